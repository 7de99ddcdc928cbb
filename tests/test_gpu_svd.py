"""The rank-r SVD compensator rule (lq_config.comp_rule = LQ_COMP_SVD) on the
GPU against the oracle's ``quantize(..., rule="svd")`` / ``commit(...,
rule="svd")``.

The r largest singular triplets of a state are unique only where the
singular values are separated; for the random states here the values after
the outlier triplets lie within a fraction of a percent of each other, so a
vector of that cluster is any unit vector of an ill-defined subspace.  The
tests therefore compare what is unique (several results are correct):

* every singular value s_c = |u_c| (relative 1e-3);
* the residual energy |S - sum_c u_c k~_c^T|_F^2 against the optimum
  sum_{c >= r} s_c^2 of Eckart-Young (never below it; at most 1e-4 above);
* for triplets separated from both neighbours by more than 5 %, k~_c itself
  (sign convention included), and u_c = S k~_c for every c;
* that the k~_c are orthonormal;
* that the snapshot is a valid quantization of the state: the dequantized
  residual plus the rank-one compensators reproduces S within half a code
  step (sigma_i c_j / 2) per element;
* decode outputs anchored on the GPU's own snapshot, against the oracle's
  window on that snapshot (exact parity, as for the row rule)."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import compare_outputs, download_snapshot, heads_major, io_dtype, oracle_tokens

pytestmark = pytest.mark.gpu

SV_RTOL = 1e-3      # singular values (the bulk cluster's Ritz values)
SEP = 1.05          # separated triplets: ratios to both neighbours above this
VEC_TOL = 1e-5      # 1 - cos of separated k~_c
ENERGY_RTOL = 1e-4  # residual energy above the Eckart-Young optimum
ORTH_TOL = 1e-5


def _cfg(B, H, dk, dv, r, gate="scalar", io="bf16", W=4, bits=8):
    return lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=W, n_comp=r,
                     gate=lq.LQ_GATE_DIAG if gate == "diag" else lq.LQ_GATE_SCALAR,
                     io_dtype=lq.LQ_BF16 if io == "bf16" else lq.LQ_F32, auto_commit=0,
                     bits=bits, comp_rule=lq.LQ_COMP_SVD)


def check_svd_snapshot(snap: dict, S: np.ndarray, r: int, what: str):
    """snap: the device snapshot (numpy, one head axis); S [nh, dv, dk]: the
    state it quantizes (FP64 or FP32)."""
    S = np.asarray(S, np.float64)
    nh = S.shape[0]
    cu_r, ck_r, sv = oracle.svd_compensators(S.astype(np.float32), r)
    for h in range(nh):
        U = snap["comp_u"][h].astype(np.float64)      # [r, dv]
        K = snap["comp_val"][h].astype(np.float64)    # [r, dk]
        s_gpu = np.linalg.norm(U, axis=1)
        s_ref = sv[h, :r]
        np.testing.assert_allclose(s_gpu, s_ref, rtol=SV_RTOL, atol=1e-6 * sv[h, 0],
                                   err_msg=f"{what} head {h}: singular values")
        assert np.abs(K @ K.T - np.eye(r)).max() <= ORTH_TOL, f"{what} head {h}: k~ not orthonormal"
        e_ref = float(np.sum(sv[h, r:] ** 2))
        e_gpu = float(np.sum((S[h] - U.T @ K) ** 2))
        scale = float(np.sum(sv[h] ** 2))
        assert e_gpu >= e_ref - 1e-6 * scale, f"{what} head {h}: residual below the optimum"
        assert e_gpu <= e_ref + ENERGY_RTOL * max(e_ref, 1e-12 * scale) + 1e-9 * scale, \
            f"{what} head {h}: residual energy {e_gpu:.6e} vs optimum {e_ref:.6e}"
        # u_c = S k~_c for every c (FP32 products of the device's k~_c)
        SK = S[h] @ K.T  # [dv, r]
        for c in range(r):
            assert np.linalg.norm(U[c] - SK[:, c]) <= 1e-5 * sv[h, 0], f"{what} head {h}: u_{c} != S k~_{c}"
        full = np.concatenate([sv[h], [0.0]])
        for c in range(r):
            left = c == 0 or full[c - 1] > SEP * full[c]
            right = full[c] > SEP * full[c + 1]
            if not (left and right):
                continue
            # a separated triplet: k~_c itself, sign included (u_c follows
            # from k~_c through S, which amplifies any residual component
            # along the largest singular direction by s_1)
            cos = float(K[c] @ ck_r[h, c])
            assert 1.0 - cos <= VEC_TOL, f"{what} head {h}: k~_{c} cos {cos}"
        # a valid quantization of S
        one = {k: v[h:h + 1] for k, v in snap.items()}
        S_hat = oracle.dequantize(one)[0]
        step = 0.5 * snap["row_scale"][h][:, None].astype(np.float64) * snap["col_smooth"][h][None, :]
        if "dense" in snap:  # BF16 residual: half a BF16 step of the residual
            step = np.abs(snap["dense"][h]).astype(np.float64) * 2.0 ** -8
        slack = 1e-5 * np.abs(S[h]).max()
        err = np.abs(S_hat - S[h])
        assert np.all(err <= step * (1 + 1e-5) + slack), \
            f"{what} head {h}: reconstruction error {float((err - step).max()):.3e} above half a step"


@pytest.mark.parametrize("dk,dv,r,bits", [(128, 128, 4, 8), (128, 128, 8, 8), (64, 128, 4, 8),
                                           (128, 64, 4, 4), (128, 128, 4, 16), (64, 64, 1, 8)])
def test_svd_init_matches_oracle(dk, dv, r, bits):
    B, H = 2, 3
    cfg = _cfg(B, H, dk, dv, r, bits=bits)
    st = lq.State(cfg, "cuda")
    S0 = synth.initial_state(0, np.arange(B), np.arange(H), dk, dv, max(1, dv // 100), max(1, dk // 100),
                             30.0).reshape(B * H, dv, dk)
    lq.lq_state_init(st, torch.from_numpy(S0).to("cuda"))
    torch.cuda.synchronize()
    snap = download_snapshot(st)
    assert np.all(snap["comp_row"] == 0)
    check_svd_snapshot(snap, S0, r, f"init d_k={dk} d_v={dv} r={r} bits={bits}")
    assert lq.lq_device_errors() == 0


def test_svd_zero_state():
    cfg = _cfg(1, 2, 128, 128, 4)
    st = lq.State(cfg, "cuda")
    st.snap.t["comp_u"].fill_(3.0)
    lq.lq_state_init(st, None)
    torch.cuda.synchronize()
    snap = download_snapshot(st)
    assert np.all(snap["comp_u"] == 0) and np.all(snap["codes"] == 0)
    assert np.all(oracle.dequantize(snap) == 0)


@pytest.mark.parametrize("dk,dv,gate,io,W,r", [(128, 128, "scalar", "bf16", 4, 4),
                                               (128, 128, "diag", "fp32", 3, 4),
                                               (64, 128, "scalar", "fp32", 5, 2),
                                               (128, 128, "scalar", "bf16", 16, 4)])
def test_svd_windows_decode_and_commit(dk, dv, gate, io, W, r):
    """Two windows: decode outputs against the oracle's window on the GPU's
    snapshot (exact parity), then the GPU's commit against the oracle's
    rebuilt state (unique parts and validity)."""
    B, H = 2, 3
    cfg = _cfg(B, H, dk, dv, r, gate, io, W)
    st = lq.State(cfg, "cuda")
    wl = synth.DecodeWorkload(f"svd_{dk}_{dv}_{gate}", B, H, dk, dv, 2 * W, W, r, gate, io, True,
                              max(1, dv // 100), max(1, dk // 100), 30.0)
    bs, hs = np.arange(B), np.arange(H)
    S0 = synth.initial_state(wl.seed, bs, hs, dk, dv, wl.outlier_rows, wl.outlier_cols,
                             wl.outlier_scale).reshape(B * H, dv, dk)
    lq.lq_state_init(st, torch.from_numpy(S0).to("cuda"))
    gdim = dk if gate == "diag" else 1
    for w in range(2):
        anchor = download_snapshot(st)
        tok = synth.tokens(wl.seed, bs, hs, w * W, (w + 1) * W, dk, dv, gate, io)
        tt = {k: torch.from_numpy(np.ascontiguousarray(v)).to("cuda") for k, v in tok.items()}
        o = torch.empty((B, W, H, dv), dtype=io_dtype(io), device="cuda")
        lq.lq_decode_window(st, tt["q"].to(io_dtype(io)), tt["k"].to(io_dtype(io)), tt["v"].to(io_dtype(io)),
                            tt["alpha"], tt["beta"], W, o)
        torch.cuda.synchronize()
        d, kt, bb, vv, qq = oracle_tokens(tok, gate)
        rec = oracle.empty_records(B * H, W, dk, dv, gdim)
        o_ref = oracle.window(anchor, rec, 0, d, kt, bb, vv, qq)
        compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, io, f"window {w}")
        S_W = oracle.rebuild(anchor, rec, W)
        lq.lq_window_commit(st)
        torch.cuda.synchronize()
        check_svd_snapshot(download_snapshot(st), S_W, r, f"commit of window {w}")
    assert lq.lq_device_errors() == 0


def test_svd_ragged_aligned_equals_synchronous():
    """Per-sequence positions started together: the ragged decode and its
    commits give exactly the synchronous path's snapshots and outputs."""
    B, H, dk, dv, W, r = 3, 2, 128, 128, 4, 4
    cfg = _cfg(B, H, dk, dv, r, W=W)
    S0 = synth.initial_state(5, np.arange(B), np.arange(H), dk, dv, 1, 1, 30.0).reshape(B * H, dv, dk)
    a, b = lq.State(cfg, "cuda"), lq.State(cfg, "cuda")
    for st in (a, b):
        lq.lq_state_init(st, torch.from_numpy(S0).to("cuda"))
    seq_pos = torch.zeros((B,), dtype=torch.int32, device="cuda")
    for t in range(W + 2):
        tok = synth.torch_tokens(5, B, H, t, t + 1, dk, dv, "scalar", "bf16", "cuda")
        oa = torch.empty((B, 1, H, dv), dtype=torch.bfloat16, device="cuda")
        ob = torch.empty_like(oa)
        lq.lq_decode_window(a, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], 1, oa)
        if a.pos == W:
            lq.lq_window_commit(a)
        lq.lq_decode_ragged(b, seq_pos, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], ob)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob), f"token {t}"
    lq.lq_ragged_flush(b, seq_pos)
    lq.lq_window_commit(a)
    torch.cuda.synchronize()
    for key in a.snap.t:
        assert torch.equal(a.snap.t[key], b.snap.t[key]), key
    assert lq.lq_device_errors() == 0


def test_svd_prefill_snapshot_is_valid():
    """The prefill's snapshot of its final FP32 state under the SVD rule."""
    B, H, dk, dv, r, T = 1, 2, 128, 128, 4, 128
    cfg = _cfg(B, H, dk, dv, r)
    st = lq.State(cfg, "cuda")
    lq.lq_state_init(st, None)
    tok = synth.torch_tokens(9, B, H, 0, T, dk, dv, "scalar", "bf16", "cuda")
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device="cuda")
    snap = lq.Snapshot(cfg, "cuda")
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    lq.lq_prefill_chunk(st, S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], T, T, [snap], o)
    torch.cuda.synchronize()
    from lqtest import snapshot_to_host
    check_svd_snapshot(snapshot_to_host(cfg, snap), S.cpu().numpy(), r, "prefill snapshot")
    for key in snap.t:
        assert torch.equal(snap.t[key], st.snap.t[key]), key
    assert lq.lq_device_errors() == 0
