"""DeltaProduct ("LeapQuant: Efficient Linear Attention with Accurate
Recurrent State Quantization", Table 4 caption: n delta-rule sub-steps per
token, each an instance of equation 1) through lq_decode_window as n
micro-tokens per token, against the oracle's deltaproduct_instance: the
outputs of each token's last sub-step and the committed snapshot."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq

from lqtest import compare_outputs, compare_snapshots, download_snapshot

pytestmark = pytest.mark.gpu


def _device_layout(x, B, H):
    """head-major [B*H, T, d] -> [B, T, H, d] (contiguous float32)."""
    x = np.asarray(x, np.float32)
    nh, T = x.shape[:2]
    y = x.reshape((B, H, T) + x.shape[2:])
    return torch.from_numpy(np.ascontiguousarray(np.swapaxes(y, 1, 2))).cuda()


@pytest.mark.parametrize("n,T,dk,dv,r", [(2, 8, 128, 128, 2), (3, 5, 64, 128, 1)])
def test_deltaproduct_micro_tokens(n, T, dk, dv, r):
    B, H = 2, 3
    nh, W = B * H, n * T
    rng = np.random.default_rng(50 + n)
    S0 = rng.normal(size=(nh, dv, dk)).astype(np.float32)
    alpha = rng.uniform(0.6, 1.0, size=(nh, T))
    beta = rng.uniform(0.1, 1.0, size=(nh, T, n))
    k = rng.normal(size=(nh, T, n, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(nh, T, n, dv))
    q = rng.normal(size=(nh, T, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    # FP32 inputs, the same values on both sides
    alpha, beta, k, v, q = (np.asarray(a, np.float32).astype(np.float64) for a in (alpha, beta, k, v, q))
    d, kt, b, vm = oracle.deltaproduct_instance(alpha, beta, k, v)
    qm = np.repeat(q, n, axis=1)
    # device micro-tokens: the gate on each token's first sub-step, beta per sub-step
    g = np.ones((nh, T, n))
    g[:, :, 0] = alpha
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=W, n_comp=r, io_dtype=lq.LQ_F32)
    st = lq.State(cfg)
    lq.lq_state_init(st, torch.from_numpy(S0).cuda())
    o = torch.empty((B, W, H, dv), dtype=torch.float32, device="cuda")
    lq.lq_decode_window(st, _device_layout(qm, B, H), _device_layout(k.reshape(nh, W, dk), B, H),
                        _device_layout(vm, B, H), _device_layout(g.reshape(nh, W), B, H),
                        _device_layout(beta.reshape(nh, W), B, H), W, o)
    torch.cuda.synchronize()
    assert st.pos == 0  # the window filled and was committed
    snap0 = oracle.quantize(S0, r)
    rec = oracle.empty_records(nh, W, dk, dv, 1)
    o_ref = oracle.window(snap0, rec, 0, d, kt, b, vm, qm)
    o_gpu = np.swapaxes(o.cpu().numpy(), 1, 2).reshape(nh, W, dv)
    last = np.arange(n - 1, W, n)  # each token's last sub-step
    compare_outputs(o_gpu[:, last], o_ref[:, last], "fp32", "DeltaProduct token outputs")
    new, _ = oracle.commit(snap0, rec, W, r)
    compare_snapshots(download_snapshot(st), new, new["row_norm"])
    assert lq.lq_device_errors() == 0
