"""Pins of the CPU oracle against what the pages and the mathematics fix.

No GPU.  Every test here ties an oracle function to something other than the
oracle itself: a published model update (Table 4 of "LeapQuant: Efficient
Linear Attention with Accurate Recurrent State Quantization"), exact rational
arithmetic, a closed form, an invariant of the quantizer, or a hand-worked
case.  Shapes use d_v != d_k so that a transposed operand fails loudly.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from linear_attention_recurrent_int8_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


# --------------------------------------------------------------------------
# Table 4: every row is an instance of equation 1
# --------------------------------------------------------------------------

def _table4_rows():
    rows = []
    with open(os.path.join(GOLDEN, "table4_eq1_instances.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([c.strip() for c in line.split("|")])
    return rows


def _published_step(model, S, alpha, beta, gamma, k, v):
    """One step of each model's own published state update, in the
    d_v x d_k orientation (row = value channel), written independently of
    equation 1."""
    dk = k.shape[0]
    I = np.eye(dk)
    if model == "linear_attention":      # Katharopoulos et al. 2020
        return S + np.outer(v, k)
    if model == "retnet":                # Sun et al. 2023, fixed decay gamma
        return gamma * S + np.outer(v, k)
    if model == "mamba2":                # Dao & Gu 2024, scalar decay per token
        return alpha[0] * S + np.outer(v, k)
    if model == "gla":                   # Yang et al. 2023, per-channel decay
        return S @ np.diag(alpha) + np.outer(v, k)
    if model == "deltanet":              # Schlag et al. 2021 delta rule
        return S @ (I - beta * np.outer(k, k)) + beta * np.outer(v, k)
    if model == "gated_deltanet":        # Yang, Kautz & Hatamizadeh 2024
        return alpha[0] * S @ (I - beta * np.outer(k, k)) + beta * np.outer(v, k)
    raise KeyError(model)


def _instance(D, KT, B, alpha, beta, gamma, k):
    dk = k.shape[0]
    d = {"I": np.ones(dk), "gamma*I": np.full(dk, gamma), "alpha*I": np.full(dk, alpha[0]),
         "Diag(alpha)": alpha}[D]
    kt = {"k": k, "beta*k": beta * k}[KT]
    b = {"0": np.zeros(dk), "k": k, "alpha*k": alpha[0] * k}[B]
    return d, kt, b


@pytest.mark.parametrize("row", _table4_rows(), ids=lambda r: r[0])
def test_table4_rows_are_instances_of_eq1(row):
    model, D, KT, B, _ = row
    dv, dk, n = 4, 5, 7
    r = _rng(1)
    S = r.normal(size=(dv, dk))
    gamma = 0.9
    ds, kts, bs, vs, qs = [], [], [], [], []
    S_pub = S.copy()
    for _ in range(n):
        alpha = 1.0 / (1.0 + np.exp(r.normal(size=dk)))
        if D != "Diag(alpha)":
            alpha = np.full(dk, alpha[0])
        beta = 1.0 / (1.0 + np.exp(-r.normal()))
        k = _unit(r.normal(size=dk))
        v = r.normal(size=dv)
        d, kt, b = _instance(D, KT, B, alpha, beta, gamma, k)
        ds.append(d), kts.append(kt), bs.append(b), vs.append(v), qs.append(r.normal(size=dk))
        S_pub = _published_step(model, S_pub, alpha, beta, gamma, k, v)
    o, S_eq1 = oracle.eq1_steps(S[None], np.array(ds)[None], np.array(kts)[None],
                                np.array(bs)[None], np.array(vs)[None], np.array(qs)[None])
    assert _rel(S_eq1[0], S_pub) < 1e-13
    # o_t = S_t q_t at the last step
    assert _rel(o[0, -1], S_pub @ qs[-1]) < 1e-13


@pytest.mark.parametrize("row", _table4_rows(), ids=lambda r: r[0])
def test_table4_record_sizes(row):
    """The buffered record of a window holds exactly Table 4's values:
    the gate only when it varies per token (1 for a scalar gate, d_k for a
    diagonal one), then k~ (d_k) and u (d_v)."""
    model, D, _, _, size = row
    dv, dk = 3, 6
    gdim = {"I": 0, "gamma*I": 0, "alpha*I": 1, "Diag(alpha)": dk}[D]
    rec = oracle.empty_records(1, 4, dk, dv, max(gdim, 1))
    per_position = (gdim if gdim else 0) + rec["k"].shape[2] + rec["u"].shape[2]
    assert per_position == eval(size.replace("d_k", str(dk)).replace("d_v", str(dv)))


def test_gated_deltanet_instance_matches_textbook():
    """oracle.gdn_instance + eq1 = alpha S (I - beta k k^T) + beta v k^T."""
    dv, dk, n = 3, 5, 9
    r = _rng(2)
    S = r.normal(size=(1, dv, dk))
    alpha = 1 / (1 + np.exp(r.normal(size=(1, n))))
    beta = 1 / (1 + np.exp(-r.normal(size=(1, n))))
    k = _unit(r.normal(size=(1, n, dk)))
    v = r.normal(size=(1, n, dv))
    q = r.normal(size=(1, n, dk))
    d, kt, b = oracle.gdn_instance(alpha, beta, k)
    o, Sn = oracle.eq1_steps(S, d, kt, b, v, q)
    X = S[0].copy()
    for t in range(n):
        X = alpha[0, t] * X @ (np.eye(dk) - beta[0, t] * np.outer(k[0, t], k[0, t])) \
            + beta[0, t] * np.outer(v[0, t], k[0, t])
        assert _rel(o[0, t], X @ q[0, t]) < 1e-13
    assert _rel(Sn[0], X) < 1e-13


def test_kda_instance_matches_published_form():
    """Kimi Delta Attention (Kimi Linear, 2025) updates S_kda (d_k x d_v) as
    (I - beta k k^T) Diag(alpha) S_kda + beta k v^T.  In the d_v x d_k
    orientation that is S Diag(alpha) (I - beta k k^T) + beta v k^T."""
    dv, dk, n = 4, 3, 8
    r = _rng(3)
    S_kda = r.normal(size=(dk, dv))
    alpha = 1 / (1 + np.exp(r.normal(size=(1, n, dk))))
    beta = 1 / (1 + np.exp(-r.normal(size=(1, n))))
    k = _unit(r.normal(size=(1, n, dk)))
    v = r.normal(size=(1, n, dv))
    d, kt, b = oracle.kda_instance(alpha, beta, k)
    _, Sn = oracle.eq1_steps(S_kda.T[None], d, kt, b, v)
    X = S_kda.copy()
    for t in range(n):
        kk = k[0, t]
        X = (np.eye(dk) - beta[0, t] * np.outer(kk, kk)) @ np.diag(alpha[0, t]) @ X \
            + beta[0, t] * np.outer(kk, v[0, t])
    assert _rel(Sn[0], X.T) < 1e-13


def test_plain_linear_attention_buffers_v():
    """With b = 0 (linear attention row of Table 4) the buffered update is u = v."""
    dv, dk, W = 4, 6, 5
    r = _rng(4)
    snap = oracle.quantize(r.normal(size=(1, dv, dk)), 1)
    rec = oracle.empty_records(1, W, dk, dv, 1)
    v = r.normal(size=(1, W, dv))
    oracle.window(snap, rec, 0, np.ones((1, W, 1)), _unit(r.normal(size=(1, W, dk))),
                  np.zeros((1, W, dk)), v, r.normal(size=(1, W, dk)))
    assert np.array_equal(rec["u"][0], v[0].astype(np.float32).astype(np.float64))


# --------------------------------------------------------------------------
# Buffered window == exact unrolled product (rational arithmetic, tiny heads)
# --------------------------------------------------------------------------

def _F(x):
    return Fraction(float(x))


def _fmat(a):
    return [[_F(x) for x in row] for row in np.atleast_2d(a)]


def _mm(A, B):
    return [[sum(A[i][k] * B[k][j] for k in range(len(B))) for j in range(len(B[0]))]
            for i in range(len(A))]


def _madd(A, B):
    return [[A[i][j] + B[i][j] for j in range(len(A[0]))] for i in range(len(A))]


def _outer(u, w):
    return [[a * b for b in w] for a in u]


def _exact_snapshot_state(snap):
    codes, rs, cs = snap["codes"][0], snap["row_scale"][0], snap["col_smooth"][0]
    dv, dk = codes.shape
    S = [[_F(rs[i]) * int(codes[i, j]) * _F(cs[j]) for j in range(dk)] for i in range(dv)]
    for c, row in enumerate(snap["comp_row"][0]):
        for j in range(dk):
            S[row][j] += _F(snap["comp_val"][0, c, j])
    return S


@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_window_equals_exact_unrolled_product(gate):
    """S_W = S^_0 prod_j (D_j - b_j k~_j^T) + sum_i v_i k~_i^T prod_{j>i}(D_j - b_j k~_j^T),
    evaluated in exact rational arithmetic, against the buffered form (records
    kept in FP64)."""
    dv, dk, W, r_c = 2, 3, 3, 1
    r = _rng(5 if gate == "scalar" else 6)
    snap = oracle.quantize(r.normal(size=(1, dv, dk)) * 2.0, r_c)
    k = _unit(r.normal(size=(1, W, dk)))
    q = r.normal(size=(1, W, dk))
    v = r.normal(size=(1, W, dv))
    beta = 1 / (1 + np.exp(-r.normal(size=(1, W))))
    if gate == "scalar":
        alpha = 1 / (1 + np.exp(r.normal(size=(1, W))))
        d, kt, b = oracle.gdn_instance(alpha, beta, k)
    else:
        alpha = 1 / (1 + np.exp(r.normal(size=(1, W, dk))))
        d, kt, b = oracle.kda_instance(alpha, beta, k)
    gdim = d.shape[2]
    rec = oracle.empty_records(1, W, dk, dv, gdim)
    o = oracle.window(snap, rec, 0, d, kt, b, v, q, exact=True)
    S_rebuilt = oracle.rebuild(snap, rec, W)

    S0 = _exact_snapshot_state(snap)
    Ms = []
    for t in range(W):
        dd = np.broadcast_to(d[0, t], (dk,))
        M = [[(_F(dd[i]) if i == j else Fraction(0)) - _F(b[0, t, i]) * _F(kt[0, t, j])
              for j in range(dk)] for i in range(dk)]
        Ms.append(M)
    for t in range(1, W + 1):
        St = S0
        for j in range(t):
            St = _mm(St, Ms[j])
        for i in range(t):
            term = _outer([_F(x) for x in v[0, i]], [_F(x) for x in kt[0, i]])
            for j in range(i + 1, t):
                term = _mm(term, Ms[j])
            St = _madd(St, term)
        o_exact = [float(sum(St[i][j] * _F(q[0, t - 1, j]) for j in range(dk))) for i in range(dv)]
        assert _rel(o[0, t - 1], o_exact) < 1e-12
    S_exact = np.array([[float(x) for x in row] for row in St])
    assert _rel(S_rebuilt[0], S_exact) < 1e-12


# --------------------------------------------------------------------------
# Buffered window == explicit stepping of the dequantized boundary state
# --------------------------------------------------------------------------

def _config1_like(gate="scalar", T=16, dk=64, dv=48, nh=3, io="fp32"):
    bs, hs = np.arange(nh), np.arange(1)
    tok = synth.tokens(0, bs, hs, 0, T, dk, dv, gate, io)
    S0 = synth.initial_state(0, bs, hs, dk, dv, 2, 0, 50.0)[:, 0]
    sq = lambda a: np.ascontiguousarray(a[:, :, 0])
    q, k, v = sq(tok["q"]), sq(tok["k"]), sq(tok["v"])
    alpha = sq(tok["alpha"])
    beta = sq(tok["beta"])
    if gate == "scalar":
        d, kt, b = oracle.gdn_instance(alpha, beta, k)
    else:
        d, kt, b = oracle.kda_instance(alpha, beta, k)
    return S0, d, kt, b, v, q


@pytest.mark.parametrize("bits", [8, 16])
@pytest.mark.parametrize("exact,tol", [(True, 1e-11), (False, 1e-5)])
@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_window_equals_explicit_stepping(gate, exact, tol, bits):
    """In-window outputs from the fixed S^_0 plus buffered updates equal
    explicitly stepping S^_0 ([LQ] Figure 2).  With FP64 records the two
    agree to rounding of FP64; with FP32 records the gap is the records'
    rounding (a few 1e-7 of the terms, relative to an output that the gate
    has shrunk)."""
    S0, d, kt, b, v, q = _config1_like(gate)
    W = d.shape[1]
    snap = oracle.quantize(S0, 4, bits=bits)
    rec = oracle.empty_records(S0.shape[0], W, S0.shape[2], S0.shape[1], d.shape[2])
    o_buf = oracle.window(snap, rec, 0, d, kt, b, v, q, exact=exact)
    o_exp, S_exp = oracle.eq1_steps(oracle.dequantize(snap), d, kt, b, v, q)
    for h in range(S0.shape[0]):
        for t in range(W):
            assert _rel(o_buf[h, t], o_exp[h, t]) < tol
    assert _rel(oracle.rebuild(snap, rec, W), S_exp) < tol


def test_window_split_calls_equal_one_call():
    """Decoding a window in pieces (pos > 0) gives the same records and outputs."""
    S0, d, kt, b, v, q = _config1_like("scalar")
    W = d.shape[1]
    snap = oracle.quantize(S0, 4)
    nh, dv, dk = S0.shape
    rec1 = oracle.empty_records(nh, W, dk, dv, 1)
    o1 = oracle.window(snap, rec1, 0, d, kt, b, v, q)
    rec2 = oracle.empty_records(nh, W, dk, dv, 1)
    parts = []
    for a, e in ((0, 5), (5, 6), (6, W)):
        sl = slice(a, e)
        parts.append(oracle.window(snap, rec2, a, d[:, sl], kt[:, sl], b[:, sl], v[:, sl], q[:, sl]))
    assert np.array_equal(np.concatenate(parts, axis=1), o1)
    for key in ("L", "k", "u"):
        assert np.array_equal(rec1[key], rec2[key])


# --------------------------------------------------------------------------
# Quantization disabled == exact recurrence
# --------------------------------------------------------------------------

@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_quantization_off_equals_recurrence(gate):
    """With every row a compensator (r = d_v) nothing is quantized: the int8
    residual is zero and each commit keeps the state in FP32.  The windowed
    chain must then follow the FP64 recurrence up to FP32 rounding."""
    S0, d, kt, b, v, q = _config1_like(gate, T=64, dv=24)
    nh, dv, dk = S0.shape
    snap = oracle.quantize(S0, dv)
    assert not snap["codes"].any()
    o_win, snap_end = oracle.decode_run(snap, d, kt, b, v, q, W=16, n_comp=dv)
    o_rec, S_rec = oracle.eq1_steps(S0.astype(np.float64), d, kt, b, v, q)
    for h in range(nh):
        for t in range(q.shape[1]):
            assert _rel(o_win[h, t], o_rec[h, t]) < 1e-5
    assert _rel(oracle.dequantize(snap_end), S_rec) < 1e-5


# --------------------------------------------------------------------------
# W = 1 and r = 0 is per-token quantization
# --------------------------------------------------------------------------

def test_w1_r0_is_per_token_quantization():
    """A loop written here from the per-token definition ([LQ] Figure 2:
    re-quantize the full state after every update): dequantize, one step of
    the recurrence, output, quantize."""
    S0, d, kt, b, v, q = _config1_like("scalar", T=24)
    nh, dv, dk = S0.shape
    snap0 = oracle.quantize(S0, 0)
    o_win, snap_win = oracle.decode_run(snap0, d, kt, b, v, q, W=1, n_comp=0)

    snap = snap0
    for t in range(q.shape[1]):
        S = (snap["row_scale"][:, :, None].astype(np.float64) * snap["codes"]
             * snap["col_smooth"][:, None, :].astype(np.float64))
        u = v[:, t] - np.einsum("hij,hj->hi", S, b[:, t])
        S = S * d[:, t][:, None, :] + u[:, :, None] * kt[:, t][:, None, :]
        o_t = np.einsum("hij,hj->hi", S, q[:, t])
        assert _rel(o_win[:, t], o_t) < 1e-6
        snap = oracle.quantize(S.astype(np.float32), 0)
    assert np.abs(snap["codes"].astype(int) - snap_win["codes"]).max() <= 1
    assert np.mean(snap["codes"] == snap_win["codes"]) > 0.999
    np.testing.assert_allclose(snap["row_scale"], snap_win["row_scale"], rtol=1e-5)


# --------------------------------------------------------------------------
# Quantizer
# --------------------------------------------------------------------------

def _outlier_state(nh=4, dv=40, dk=24, seed=7):
    r = _rng(seed)
    S = r.normal(size=(nh, dv, dk))
    S[:, 3, :] *= 30
    S[:, :, 5] *= 30
    S[:, 11, :] *= 8
    return S.astype(np.float32)


@pytest.mark.parametrize("bits", [8, 6, 4])
@pytest.mark.parametrize("smoothing", [True, False])
@pytest.mark.parametrize("r", [0, 1, 4])
def test_quantizer_error_bound_and_compensators(r, smoothing, bits):
    """Round to nearest: every residual element is within half a code step
    (sigma_i c_j / 2) of the original, at every code width."""
    S = _outlier_state()
    snap = oracle.quantize(S, r, smoothing, bits)
    S_hat = oracle.dequantize(snap)
    sig = snap["row_scale"].astype(np.float64)
    c = snap["col_smooth"].astype(np.float64)
    bound = 0.5 * sig[:, :, None] * c[:, None, :] * (1 + 1e-6) + 1e-30
    for h in range(S.shape[0]):
        comp = set(snap["comp_row"][h].tolist())
        assert len(comp) == r
        for i in range(S.shape[1]):
            if i in comp:
                # compensator rows are held exactly
                assert np.array_equal(S_hat[h, i], S[h, i].astype(np.float64))
            else:
                assert np.all(np.abs(S[h, i] - S_hat[h, i]) <= bound[h, i])


@pytest.mark.parametrize("r", [1, 3, 8])
def test_quantizer_selects_top_r_rows(r):
    S = _outlier_state(seed=8)
    snap = oracle.quantize(S, r)
    norms = np.linalg.norm(S.astype(np.float64), axis=2)
    for h in range(S.shape[0]):
        order = sorted(range(S.shape[1]), key=lambda i: (-norms[h, i], i))
        assert snap["comp_row"][h].tolist() == order[:r]
        residual = np.delete(norms[h], order[:r])
        # the residual's largest row norm is the (r+1)-th largest original one
        assert residual.max() == norms[h, order[r]]
    np.testing.assert_allclose(snap["row_norm"], norms, rtol=1e-15)


@pytest.mark.parametrize("bits,qmax", [(8, 127), (6, 31), (4, 7)])
def test_quantizer_smoothing_and_code_range(bits, qmax):
    S = _outlier_state(seed=9)
    r = 2
    snap = oracle.quantize(S, r, bits=bits)
    for h in range(S.shape[0]):
        R = S[h].astype(np.float64).copy()
        R[snap["comp_row"][h]] = 0
        m = np.abs(R).max(axis=0)
        c = snap["col_smooth"][h].astype(np.float64)
        # c_j = sqrt(max_i |R_ij|), rounded once to FP32
        np.testing.assert_array_equal(c, np.sqrt(m).astype(np.float32))
        assert np.all(np.abs(c * c - m) <= 2.0 ** -22 * m)
        codes = snap["codes"][h].astype(int)
        nz = snap["row_scale"][h] > 0
        # every nonzero row reaches the end of the code range, none passes it
        assert np.all(np.abs(codes[nz]).max(axis=1) == qmax)
        assert codes.min() >= -qmax and codes.max() <= qmax
        assert not codes[~nz].any()
        # sigma = row max / qmax: the largest code reconstructs the row max
        Rp = R / snap["col_smooth"][h].astype(np.float64)[None, :]
        np.testing.assert_allclose(snap["row_scale"][h][nz] * qmax,
                                   np.abs(Rp).max(axis=1)[nz], rtol=2e-7)


def test_quantizer_hand_cases():
    dv, dk = 6, 8
    # zero state: no scale, unit smoothing, ties to the smallest rows
    z = oracle.quantize(np.zeros((1, dv, dk), np.float32), 3)
    assert not z["codes"].any() and not z["row_scale"].any() and not z["comp_val"].any()
    assert np.all(z["col_smooth"] == 1.0)
    assert z["comp_row"][0].tolist() == [0, 1, 2]
    # a constant row quantizes to +127 everywhere
    S = np.zeros((1, dv, dk), np.float32)
    S[0, 2, :] = 0.37
    S[0, 4, 1] = -0.01
    s = oracle.quantize(S, 0, smoothing=False)
    assert np.all(s["codes"][0, 2] == 127)
    assert s["codes"][0, 4, 1] == -127
    # round half to even: sigma = 1 exactly, quotients 2.5 -> 2, -0.5 -> 0, 1.5 -> 2
    S = np.zeros((1, dv, dk), np.float32)
    S[0, 3, :4] = [127.0, 2.5, -0.5, 1.5]
    s = oracle.quantize(S, 0, smoothing=False)
    assert s["row_scale"][0, 3] == 1.0
    assert s["codes"][0, 3, :4].tolist() == [127, 2, 0, 2]
    # a single spike with smoothing: c = sqrt(spike), code 127, exact reconstruction
    S = np.zeros((1, dv, dk), np.float32)
    S[0, 1, 5] = 7.0
    s = oracle.quantize(S, 0)
    assert s["codes"][0, 1, 5] == 127
    assert s["col_smooth"][0, 5] == np.float32(np.sqrt(7.0))
    assert abs(oracle.dequantize(s)[0, 1, 5] - 7.0) < 1e-5


@pytest.mark.parametrize("bits,qmax,name", [(8, 127, "quantizer_hand_case.txt"),
                                             (6, 31, "quantizer_hand_case_6bit.txt"),
                                             (4, 7, "quantizer_hand_case_4bit.txt")])
def test_quantizer_golden_hand_case(bits, qmax, name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = [float(x) for x in rest]
    dv, dk = (int(x) for x in vals["shape"])
    S = np.array(vals["state"], np.float32).reshape(1, dv, dk)
    s = oracle.quantize(S, int(vals["n_comp"][0]), bits=bits)
    assert s["comp_row"][0].tolist() == [int(x) for x in vals["comp_row"]]
    np.testing.assert_array_equal(s["comp_val"][0].ravel(), np.float32(vals["comp_val"]))
    np.testing.assert_array_equal(s["col_smooth"][0], np.float32(vals["col_smooth"]))
    np.testing.assert_array_equal(s["codes"][0].ravel(), np.int8(vals["codes"]))
    np.testing.assert_allclose(s["row_scale"][0] * qmax, vals[f"row_scale_times_{qmax}"], rtol=1e-6)


def test_quantizer_narrow_codes_hand_cases():
    """4-bit: sigma = 1 exactly for a row of maximum 7; quotients 2.5 -> 2,
    -0.5 -> 0, 1.5 -> 2, 3.5 -> 4 (half to even), -6.5 -> -6.  6-bit: a row of
    maximum 31 likewise."""
    dv, dk = 4, 8
    S = np.zeros((1, dv, dk), np.float32)
    S[0, 1, :6] = [7.0, 2.5, -0.5, 1.5, 3.5, -6.5]
    s = oracle.quantize(S, 0, smoothing=False, bits=4)
    assert s["row_scale"][0, 1] == 1.0
    assert s["codes"][0, 1, :6].tolist() == [7, 2, 0, 2, 4, -6]
    S[0, 1, :6] = [31.0, 2.5, -0.5, 1.5, 30.5, -29.5]
    s = oracle.quantize(S, 0, smoothing=False, bits=6)
    assert s["row_scale"][0, 1] == 1.0
    assert s["codes"][0, 1, :6].tolist() == [31, 2, 0, 2, 30, -30]


def _golden_vals(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = [float(x) for x in rest]
    return vals


@pytest.mark.parametrize("name", ["quantizer_division_scale_case.txt",
                                  "quantizer_division_smoothing_case.txt"])
def test_quantizer_divides_in_fp32(name):
    """Hand-worked cases (derivations in the fixtures) whose codes differ
    between true FP32 quotients R / c and R' / sigma (the rule) and products
    with a rounded inverse factor or scale: a half-way quotient is exact in
    the first form and lands one FP32 step above the tie in the second."""
    vals = _golden_vals(name)
    dv, dk = (int(x) for x in vals["shape"])
    S = np.array(vals["state"], np.float32).reshape(1, dv, dk)
    s = oracle.quantize(S, int(vals["n_comp"][0]), smoothing=bool(vals["smoothing"][0]))
    np.testing.assert_array_equal(s["col_smooth"][0], np.float32(vals["col_smooth"]))
    np.testing.assert_array_equal(s["codes"][0].ravel(), np.int8(vals["codes"]))
    np.testing.assert_allclose(s["row_scale"][0] * 127, vals["row_scale_times_127"], rtol=1e-6)


# --------------------------------------------------------------------------
# Prefill oracle: snapshots are the quantized recurrence state
# --------------------------------------------------------------------------

def test_prefill_snapshots_are_quantized_recurrence_states():
    S0, d, kt, b, v, q = _config1_like("scalar", T=48, dv=16, dk=32, nh=2)
    S0 = np.zeros_like(S0, dtype=np.float64)
    o, snaps, S_end = oracle.prefill(S0, d, kt, b, v, q, snapshot_every=16, n_comp=2)
    assert len(snaps) == 3
    for n in range(3):
        T = 16 * (n + 1)
        _, S_T = oracle.eq1_steps(S0, d[:, :T], kt[:, :T], b[:, :T], v[:, :T], q[:, :T])
        ref = oracle.quantize(S_T.astype(np.float32), 2)
        for key in ("codes", "row_scale", "col_smooth", "comp_row", "comp_val"):
            np.testing.assert_array_equal(snaps[n][key], ref[key])
    o_ref, _ = oracle.eq1_steps(S0, d, kt, b, v, q)
    assert np.array_equal(o, o_ref)


def test_ragged_last_window_commits():
    S0, d, kt, b, v, q = _config1_like("scalar", T=21)
    snap = oracle.quantize(S0, 4)
    seen = []
    oracle.decode_run(snap, d, kt, b, v, q, W=8, n_comp=4, on_commit=lambda i, s: seen.append(i))
    assert seen == [0, 1, 2]


@pytest.mark.parametrize("diagonal", [False, True])
def test_gated_linear_instance_matches_published_updates(diagonal):
    """oracle.gated_linear_instance + eq1 = the Mamba2 (scalar decay) or GLA
    (per-channel decay) update alpha S + v k^T with beta = 1, and
    alpha S + beta v k^T in general; the outputs are S_t q_t."""
    dv, dk, n = 3, 5, 8
    r = _rng(7)
    S = r.normal(size=(dv, dk))
    nh = 1
    alpha = 1.0 / (1.0 + np.exp(r.normal(size=(nh, n, dk) if diagonal else (nh, n))))
    for beta_is_one in (True, False):
        beta = np.ones((nh, n)) if beta_is_one else 1.0 / (1.0 + np.exp(-r.normal(size=(nh, n))))
        k = np.stack([_unit(r.normal(size=dk)) for _ in range(n)])[None]
        v = r.normal(size=(nh, n, dv))
        q = r.normal(size=(nh, n, dk))
        d, kt, b = oracle.gated_linear_instance(alpha, beta, k, diagonal)
        assert np.all(b == 0.0)
        o, S_eq1 = oracle.eq1_steps(S[None], d, kt, b, v, q)
        S_pub = S.copy()
        for t in range(n):
            decay = np.diag(alpha[0, t]) if diagonal else alpha[0, t] * np.eye(dk)
            S_pub = S_pub @ decay + beta[0, t] * np.outer(v[0, t], k[0, t])
            assert _rel(o[0, t], S_pub @ q[0, t]) < 1e-13
        assert _rel(S_eq1[0], S_pub) < 1e-13


# --------------------------------------------------------------------------
# BF16 state ([LQ] Table 2, "BF16 per-step" and its per-window row)
# --------------------------------------------------------------------------

def test_bf16_state_is_round_to_nearest_even_of_the_residual():
    """The BF16 residual equals torch's float32 -> bfloat16 conversion (round
    to nearest, ties to even) of the state with its compensator rows zeroed;
    scales are 1, codes 0, compensators the top-r rows as at 8 bits."""
    import torch
    S = _outlier_state(seed=21)
    r = 3
    snap = oracle.quantize(S, r, bits=16)
    ref8 = oracle.quantize(S, r)
    for h in range(S.shape[0]):
        assert snap["comp_row"][h].tolist() == ref8["comp_row"][h].tolist()
        R = S[h].copy()
        R[snap["comp_row"][h]] = 0
        want = torch.from_numpy(R).to(torch.bfloat16).to(torch.float32).numpy()
        np.testing.assert_array_equal(snap["dense"][h], want)
        np.testing.assert_array_equal(snap["comp_val"][h], S[h][snap["comp_row"][h]])
    assert np.all(snap["row_scale"] == 1.0) and np.all(snap["col_smooth"] == 1.0)
    assert not snap["codes"].any()
    # dequantized: the BF16 residual plus the exact compensator rows
    Sh = oracle.dequantize(snap)
    for h in range(S.shape[0]):
        rows = snap["comp_row"][h]
        np.testing.assert_array_equal(Sh[h][rows], S[h][rows].astype(np.float64))
        keep = np.setdiff1d(np.arange(S.shape[1]), rows)
        np.testing.assert_array_equal(Sh[h][keep], snap["dense"][h][keep].astype(np.float64))


def test_bf16_state_hand_cases():
    """8 significant bits: 1 + 2^-8 is a tie between 1 and 1 + 2^-7 and goes
    to the even 1; 1 + 3 2^-8 goes to the even 1 + 2^-6; just above a tie
    rounds up; values with 8 bits are kept; negatives are symmetric."""
    vals = [1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, 3.0, -(1 + 2 ** -8 + 2 ** -20),
            0.0, 255.0, 257.0, 2 ** -30 * (1 + 2 ** -9)]
    want = [1.0, 1 + 2 ** -6, 1 + 2 ** -7, 3.0, -(1 + 2 ** -7), 0.0, 255.0, 256.0, 2 ** -30]
    S = np.zeros((1, 4, 16), np.float32)
    S[0, 1, :len(vals)] = vals
    snap = oracle.quantize(S, 0, bits=16)
    assert snap["dense"][0, 1, :len(vals)].tolist() == [float(np.float32(w)) for w in want]


# --------------------------------------------------------------------------
# Rank-r SVD compensators (the variant of the row rule)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("r", [1, 3, 6])
def test_svd_compensators_are_the_best_rank_r_part(r):
    """Eckart-Young: the residual S - sum_c u_c k~_c^T has spectral norm
    s_{r+1} and squared Frobenius norm sum_{c>r} s_c^2 (up to the FP32
    rounding of the factors); each pair satisfies S k~_c = u_c and
    S^T u_c = s_c^2 k~_c with |k~_c| = 1; and no rank-r row selection leaves a
    smaller residual."""
    S = _outlier_state(seed=31)
    cu, ck, sv = oracle.svd_compensators(S, r)
    for h in range(S.shape[0]):
        A = S[h].astype(np.float64)
        P = cu[h].astype(np.float64).T @ ck[h].astype(np.float64)
        R = A - P
        scale = sv[h][0]
        assert abs(np.linalg.norm(R, 2) - sv[h][r]) <= 1e-5 * scale
        assert abs(np.linalg.norm(R) ** 2 - np.sum(sv[h][r:] ** 2)) <= 1e-5 * scale ** 2
        for c in range(r):
            k = ck[h, c].astype(np.float64)
            u = cu[h, c].astype(np.float64)
            assert abs(np.linalg.norm(k) - 1.0) < 1e-6
            assert np.linalg.norm(A @ k - u) <= 1e-5 * scale
            assert np.linalg.norm(A.T @ u - sv[h][c] ** 2 * k) <= 1e-5 * scale ** 2
            assert k[np.argmax(np.abs(k))] > 0  # the sign convention
        rows = np.argsort(-np.linalg.norm(A, axis=1), kind="stable")[:r]
        Rrow = A.copy()
        Rrow[rows] = 0
        assert np.linalg.norm(R) <= np.linalg.norm(Rrow) * (1 + 1e-6)


def test_svd_rule_on_a_rank_r_state_leaves_no_residual():
    """A state of rank r is held entirely by r SVD compensators: the residual
    is FP32 rounding only, far below the state's scale."""
    rng = _rng(32)
    r, dv, dk = 3, 24, 32
    S = (rng.normal(size=(2, dv, r)) @ rng.normal(size=(2, r, dk))).astype(np.float32)
    snap = oracle.quantize(S, r, smoothing=False, rule="svd")
    # without smoothing sigma_i * 127 is the residual row's largest magnitude
    assert np.abs(snap["row_scale"]).max() * 127 <= 1e-5 * np.abs(S).max()
    np.testing.assert_allclose(oracle.dequantize(snap), S.astype(np.float64), atol=1e-5 * np.abs(S).max())


def test_svd_rule_with_no_compensators_is_the_row_rule():
    S = _outlier_state(seed=33)
    a, b = oracle.quantize(S, 0, rule="svd"), oracle.quantize(S, 0)
    for key in ("codes", "row_scale", "col_smooth"):
        np.testing.assert_array_equal(a[key], b[key])


@pytest.mark.parametrize("gate", ["scalar", "diag"])
def test_svd_compensators_share_the_update_path(gate):
    """Decoding a window from an SVD-compensated snapshot equals explicit
    stepping of its dequantized state (the compensators are pseudo-tokens at
    window position 0 with u = u_c, k~ = k~_c), and the rebuild equals the
    stepped state."""
    S0, d, kt, b, v, q = _config1_like(gate)
    W = d.shape[1]
    snap = oracle.quantize(S0, 4, rule="svd")
    rec = oracle.empty_records(S0.shape[0], W, S0.shape[2], S0.shape[1], d.shape[2])
    o_buf = oracle.window(snap, rec, 0, d, kt, b, v, q, exact=True)
    o_exp, S_exp = oracle.eq1_steps(oracle.dequantize(snap), d, kt, b, v, q)
    for h in range(S0.shape[0]):
        for t in range(W):
            assert _rel(o_buf[h, t], o_exp[h, t]) < 1e-11
    assert _rel(oracle.rebuild(snap, rec, W), S_exp) < 1e-11
    # and the dequantized state is the quantized residual plus the rank-r part
    P = np.einsum("hci,hcj->hij", snap["comp_u"].astype(np.float64), snap["comp_val"].astype(np.float64))
    res = oracle.dequantize({k2: v2 for k2, v2 in snap.items() if k2 != "comp_u"} | {
        "comp_row": np.zeros((S0.shape[0], 0), np.int32),
        "comp_val": np.zeros((S0.shape[0], 0, S0.shape[2]), np.float32)})
    np.testing.assert_allclose(oracle.dequantize(snap), res + P, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# DeltaProduct: n delta-rule sub-steps per token ([LQ] Table 4 caption)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", [1, 2, 3])
def test_deltaproduct_micro_tokens_equal_the_householder_product(n):
    """Equation 1 over the micro-tokens equals the published DeltaProduct
    update, written here with explicit matrices: S_t = alpha_t S_{t-1} H_t +
    sum_j beta_j v_j k_j^T prod_{l>j} (I - beta_l k_l k_l^T), with H_t the
    product of the n Householder-like factors (I - beta_j k_j k_j^T); the
    token's output is S_t q_t.  The window (buffered) decode of the same
    micro-tokens from a quantized state gives the same outputs as stepping
    its dequantized state."""
    rng = _rng(40 + n)
    nh, T, dk, dv = 2, 5, 6, 4
    S0 = rng.normal(size=(nh, dv, dk))
    alpha = rng.uniform(0.5, 1.0, size=(nh, T))
    beta = rng.uniform(0.1, 1.0, size=(nh, T, n))
    k = rng.normal(size=(nh, T, n, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(nh, T, n, dv))
    q = rng.normal(size=(nh, T, dk))
    d, kt, b, vm = oracle.deltaproduct_instance(alpha, beta, k, v)
    qm = np.repeat(q, n, axis=1)  # any q for the inner sub-steps; only the last output is used
    o_m, S_m = oracle.eq1_steps(S0, d, kt, b, vm, qm)
    I = np.eye(dk)
    for h in range(nh):
        S = S0[h].copy()
        for t in range(T):
            H = [I - beta[h, t, j] * np.outer(k[h, t, j], k[h, t, j]) for j in range(n)]
            P = I.copy()
            for j in range(n):
                P = P @ H[j]
            add = np.zeros((dv, dk))
            for j in range(n):
                tail = I.copy()
                for l in range(j + 1, n):
                    tail = tail @ H[l]
                add += beta[h, t, j] * np.outer(v[h, t, j], k[h, t, j]) @ tail
            S = alpha[h, t] * S @ P + add
            assert _rel(o_m[h, t * n + n - 1], S @ q[h, t]) < 1e-12
        assert _rel(S_m[h], S) < 1e-12
    # the buffered window over the micro-tokens (W = T n) equals stepping the
    # dequantized boundary state
    snap = oracle.quantize(S0.astype(np.float32), 1)
    rec = oracle.empty_records(nh, T * n, dk, dv, 1)
    o_w = oracle.window(snap, rec, 0, d, kt, b, vm, qm, exact=True)
    o_s, _ = oracle.eq1_steps(oracle.dequantize(snap), d, kt, b, vm, qm)
    for h in range(nh):
        for t in range(T):
            assert _rel(o_w[h, t * n + n - 1], o_s[h, t * n + n - 1]) < 1e-11
