"""The C-ABI library builds, loads and exports every symbol include/lq.h
declares; its host-side validation rejects bad arguments before any launch.
No GPU: nothing here reaches a kernel launch."""
import ctypes
import os
import re
import subprocess

import pytest

import linear_attention_recurrent_int8_b200 as lq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lq.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LQ_API\s+[\w\s\*]+?\b(lq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = lq.load_library()
    declared = _declared()
    assert declared == sorted(lq.ABI_SYMBOLS)
    out = subprocess.run(["nm", "-D", "--defined-only", lq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(set(re.findall(r"\bT (lq_\w+)$", out, re.M)))
    assert exported == declared
    for name in declared:
        assert getattr(lib, name) is not None


def test_status_strings():
    names = ["LQ_OK", "LQ_ERR_INVALID_ARGUMENT", "LQ_ERR_UNSUPPORTED", "LQ_ERR_WINDOW_FULL",
             "LQ_ERR_WINDOW_OPEN", "LQ_ERR_MISALIGNED", "LQ_ERR_CUDA"]
    for i, n in enumerate(names):
        assert lq.lq_status_string(i) == n
    assert lq.lq_status_string(99) == "LQ_UNKNOWN_STATUS"


def test_buffer_elems():
    cfg = lq.Config(batch=3, heads=5, d_k=128, d_v=64, window=16, n_comp=4,
                    gate=lq.LQ_GATE_DIAG)
    bh = 15
    want = [bh * 64 * 128, bh * 64, bh * 128, bh * 4, bh * 4 * 128, bh * 16 * 128,
            bh * 16 * 128, bh * 16 * 64]
    assert [lq.lq_buffer_elems(cfg, w) for w in range(8)] == want
    assert lq.lq_buffer_elems(cfg, 8) == 0  # comp_u: only with the SVD rule
    assert lq.lq_buffer_elems(cfg, 9) == -1
    cfg.comp_rule = lq.LQ_COMP_SVD
    assert lq.lq_buffer_elems(cfg, 8) == bh * 4 * 64
    cfg.comp_rule = 2
    assert lq.lq_buffer_elems(cfg, 8) == -1  # not a rule
    cfg.comp_rule = lq.LQ_COMP_ROWS
    cfg.gate = lq.LQ_GATE_SCALAR
    assert lq.lq_buffer_elems(cfg, 5) == bh * 16
    # code bytes: one per code at 8 and 6 bits (0 means 8), half a byte at 4
    for bits, want0 in ((0, bh * 64 * 128), (8, bh * 64 * 128), (6, bh * 64 * 128),
                        (4, bh * 64 * 64), (16, bh * 64 * 128)):
        cfg.bits = bits
        assert lq.lq_buffer_elems(cfg, 0) == want0, bits
    cfg.bits = 5
    assert lq.lq_buffer_elems(cfg, 0) == -1
    cfg.bits = 8
    cfg.d_k = 96
    assert lq.lq_buffer_elems(cfg, 0) == -1


def test_four_bit_packing_helpers_follow_the_header():
    """lq.h: in each group of 8 key channels 8g..8g+7 of a row, byte 4g+b
    holds channel 8g+b in its low nibble and 8g+4+b in its high nibble, two's
    complement.  Hand-packed example, then a random round trip."""
    import numpy as np
    from lqtest import pack_codes4, unpack_codes4
    row = np.array([1, 2, 3, 4, 5, 6, 7, -7, 0, -1, -8 + 1, 0, 3, -2, 0, 7], np.int8)
    packed = pack_codes4(row)
    assert packed.tolist() == [0x51, 0x62, 0x73, 0x94, 0x30, 0xEF, 0x09, 0x70]
    assert unpack_codes4(packed).tolist() == row.tolist()
    r = np.random.default_rng(0).integers(-7, 8, size=(3, 5, 64)).astype(np.int8)
    p = pack_codes4(r)
    assert p.shape == (3, 5, 32) and p.dtype == np.uint8
    assert np.array_equal(unpack_codes4(p), r)


class _Buf:
    """A fake aligned 'device' address; validation never dereferences it."""

    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _fake_state(cfg, pos=0, base=0x10000000):
    st = lq.LqState()
    st.cfg = cfg.c()
    a = [base + 0x100000 * i for i in range(8)]
    st.snap = lq.LqSnapshot(a[0], a[1], a[2], a[3], a[4])
    st.buf_gate, st.buf_k, st.buf_u = a[5], a[6], a[7]
    st.pos = pos
    st.impl = None
    return st


def _decode(st, n, q=0x20000000, o=0x21000000, stream=None):
    lib = lq.load_library()
    return lib.lq_decode_window(ctypes.byref(st), q, q + 0x100000, q + 0x200000, q + 0x300000,
                                q + 0x400000, n, o, stream)


def test_decode_validation_without_launch():
    lib = lq.load_library()
    cfg = lq.Config(batch=2, heads=3, window=4, n_comp=2)
    assert lib.lq_decode_window(None, None, None, None, None, None, 1, None, None) == \
        lq.LQ_ERR_INVALID_ARGUMENT
    # window full: pos + n > W
    assert _decode(_fake_state(cfg, pos=3), 2) == lq.LQ_ERR_WINDOW_FULL
    # n_steps == 0 is a no-op, n_steps < 0 invalid
    assert _decode(_fake_state(cfg, pos=4), 0) == lq.LQ_OK
    assert _decode(_fake_state(cfg), -1) == lq.LQ_ERR_INVALID_ARGUMENT
    # null inputs
    st = _fake_state(cfg)
    assert lib.lq_decode_window(ctypes.byref(st), None, 1, 1, 1, 1, 1, 1, None) == \
        lq.LQ_ERR_INVALID_ARGUMENT
    # misaligned state buffer
    st = _fake_state(cfg)
    st.buf_k = st.buf_k + 4
    assert _decode(st, 1) == lq.LQ_ERR_MISALIGNED
    # misaligned activations: odd address, and element-aligned but not 16-byte aligned
    assert _decode(_fake_state(cfg), 1, q=0x20000001) == lq.LQ_ERR_MISALIGNED
    assert _decode(_fake_state(cfg), 1, q=0x20000002) == lq.LQ_ERR_MISALIGNED
    # unsupported head size, bad window, too many compensators
    for field, val, want in (("d_k", 96, lq.LQ_ERR_UNSUPPORTED), ("window", 33, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("window", 0, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("n_comp", 17, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("gate", 2, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("delta", 2, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("bits", 5, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("bits", 12, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("bits", 32, lq.LQ_ERR_INVALID_ARGUMENT),
                             ("batch", 0, lq.LQ_ERR_INVALID_ARGUMENT)):
        c2 = lq.Config(batch=2, heads=3, window=4, n_comp=2)
        setattr(c2, field, val)
        assert _decode(_fake_state(c2), 1) == want, field
    # compensator pointers may be null only when n_comp == 0
    st = _fake_state(cfg)
    st.snap.comp_val = None
    assert _decode(st, 1) == lq.LQ_ERR_INVALID_ARGUMENT


def test_commit_snapshot_prefill_validation_without_launch():
    lib = lq.load_library()
    cfg = lq.Config(batch=1, heads=2, window=8, n_comp=1)
    # commit at pos == 0 is a no-op
    assert lib.lq_window_commit(ctypes.byref(_fake_state(cfg, pos=0)), None) == lq.LQ_OK
    # snapshot / restore / prefill need a closed window
    dst = lq.LqSnapshot(0x30000000, 0x30100000, 0x30200000, 0x30300000, 0x30400000)
    assert lib.lq_state_snapshot(ctypes.byref(_fake_state(cfg, pos=3)), ctypes.byref(dst), None) == \
        lq.LQ_ERR_WINDOW_OPEN
    assert lib.lq_state_restore(ctypes.byref(_fake_state(cfg, pos=3)), ctypes.byref(dst), None) == \
        lq.LQ_ERR_WINDOW_OPEN
    p = 0x40000000
    args = [p, p + 0x100000, p + 0x200000, p + 0x300000, p + 0x400000, p + 0x500000]
    st = _fake_state(cfg, pos=2)
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 128, 64, None, p + 0x600000, None, 0, None) == \
        lq.LQ_ERR_WINDOW_OPEN
    st = _fake_state(cfg)
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 0, 64, None, p + 0x600000, None, 0, None) == lq.LQ_OK
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 128, 0, None, p + 0x600000, None, 0, None) == \
        lq.LQ_ERR_INVALID_ARGUMENT
    snaps = (lq.LqSnapshot * 2)(dst, dst)
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 100, 64, snaps, p + 0x600000, None, 0, None) == \
        lq.LQ_ERR_INVALID_ARGUMENT
    # workspace: pointer and size go together; 16-byte aligned
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 128, 64, None, p + 0x600000, None, 4096,
                                None) == lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 128, 64, None, p + 0x600000, p + 0x700000,
                                0, None) == lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_prefill_chunk(ctypes.byref(st), *args, 128, 64, None, p + 0x600000, p + 0x700008,
                                4096, None) == lq.LQ_ERR_MISALIGNED
    bad = list(args)
    bad[0] += 4
    assert lib.lq_prefill_chunk(ctypes.byref(st), *bad, 128, 64, None, p + 0x600000, None, 0, None) == \
        lq.LQ_ERR_MISALIGNED
    # fp32 comparator: negative steps, null state
    c = cfg.c()
    assert lib.lq_fp32_step(ctypes.byref(c), None, *args[1:], 1, p, None) == lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_fp32_step(ctypes.byref(c), p, *args[1:], -1, p, None) == lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_fp32_step(ctypes.byref(c), p, *args[1:], 0, p, None) == lq.LQ_OK


def test_state_init_validation_without_launch():
    lib = lq.load_library()
    cfg = lq.Config(batch=1, heads=1, d_v=64, d_k=64, n_comp=65)
    st = _fake_state(lq.Config(batch=1, heads=1))
    c = cfg.c()
    assert lib.lq_state_init(ctypes.byref(st), ctypes.byref(c), None, None) == \
        lq.LQ_ERR_INVALID_ARGUMENT
    cfg.n_comp = 4
    c = cfg.c()
    assert lib.lq_state_init(ctypes.byref(st), ctypes.byref(c), 0x1234, None) == lq.LQ_ERR_MISALIGNED
    assert lib.lq_state_init(None, ctypes.byref(c), None, None) == lq.LQ_ERR_INVALID_ARGUMENT


def test_ragged_validation_without_launch():
    lib = lq.load_library()
    cfg = lq.Config(batch=2, heads=3, window=4, n_comp=2)
    p = 0x50000000
    toks = [p, p + 0x100000, p + 0x200000, p + 0x300000, p + 0x400000]
    o = p + 0x500000
    # no positions array, misaligned positions, an open synchronous window, null inputs
    assert lib.lq_decode_ragged(ctypes.byref(_fake_state(cfg)), None, *toks, o, None) == \
        lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_decode_ragged(ctypes.byref(_fake_state(cfg)), p + 0x600002, *toks, o, None) == \
        lq.LQ_ERR_MISALIGNED
    assert lib.lq_decode_ragged(ctypes.byref(_fake_state(cfg, pos=1)), p + 0x600000, *toks, o,
                                None) == lq.LQ_ERR_WINDOW_OPEN
    assert lib.lq_decode_ragged(ctypes.byref(_fake_state(cfg)), p + 0x600000, None, *toks[1:], o,
                                None) == lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_decode_ragged(None, p + 0x600000, *toks, o, None) == lq.LQ_ERR_INVALID_ARGUMENT


def test_binding_structs_match_the_header_layout(tmp_path):
    """The ctypes mirrors of lq_config, lq_snapshot and lq_state have the
    C header's field names, offsets and sizes (a C program compiled against
    include/lq.h prints them)."""
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    structs = {"lq_config": lq.LqConfig, "lq_snapshot": lq.LqSnapshot, "lq_state": lq.LqState}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "lq.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(root, "include"), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {(a, b): int(c) for a, b, c in (ln.split() for ln in out if ln.strip())}
    for cname, py in structs.items():
        assert got[(cname, "sizeof")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_per_sequence_mode_refuses_calls_that_need_closed_windows():
    """After lq_decode_ragged the state's pos is LQ_POS_PER_SEQUENCE: windows
    may be open on the device, so synchronous decode, commit, snapshot,
    restore and prefill refuse (LQ_ERR_WINDOW_OPEN) until lq_ragged_flush."""
    lib = lq.load_library()
    cfg = lq.Config(batch=2, heads=3, window=4, n_comp=2)
    per_seq = lambda: _fake_state(cfg, pos=lq.LQ_POS_PER_SEQUENCE)
    assert _decode(per_seq(), 1) == lq.LQ_ERR_WINDOW_OPEN
    assert lib.lq_window_commit(ctypes.byref(per_seq()), None) == lq.LQ_ERR_WINDOW_OPEN
    dst = lq.LqSnapshot(0x30000000, 0x30100000, 0x30200000, 0x30300000, 0x30400000)
    assert lib.lq_state_snapshot(ctypes.byref(per_seq()), ctypes.byref(dst), None) == \
        lq.LQ_ERR_WINDOW_OPEN
    assert lib.lq_state_restore(ctypes.byref(per_seq()), ctypes.byref(dst), None) == \
        lq.LQ_ERR_WINDOW_OPEN
    p = 0x40000000
    args = [p, p + 0x100000, p + 0x200000, p + 0x300000, p + 0x400000, p + 0x500000]
    assert lib.lq_prefill_chunk(ctypes.byref(per_seq()), *args, 128, 64, None, p + 0x600000,
                                None, 0, None) == lq.LQ_ERR_WINDOW_OPEN
    # other negative positions stay invalid
    assert _decode(_fake_state(cfg, pos=-2), 1) == lq.LQ_ERR_INVALID_ARGUMENT
    # the flush: positions array required and aligned; an open synchronous window refuses
    assert lib.lq_ragged_flush(ctypes.byref(per_seq()), None, None) == lq.LQ_ERR_INVALID_ARGUMENT
    assert lib.lq_ragged_flush(ctypes.byref(per_seq()), p + 2, None) == lq.LQ_ERR_MISALIGNED
    assert lib.lq_ragged_flush(ctypes.byref(_fake_state(cfg, pos=3)), p, None) == \
        lq.LQ_ERR_WINDOW_OPEN
    assert lib.lq_ragged_flush(None, p, None) == lq.LQ_ERR_INVALID_ARGUMENT


def test_batch_times_heads_is_bounded():
    """B * H <= 2^24 keeps every grid and per-head index inside 2^31."""
    cfg = lq.Config(batch=1 << 12, heads=1 << 12, window=4, n_comp=2)
    assert lq.lq_buffer_elems(cfg, 1) == (1 << 24) * 128
    cfg.heads = (1 << 12) + 1
    assert lq.lq_buffer_elems(cfg, 1) == -1
    assert _decode(_fake_state(cfg), 1) == lq.LQ_ERR_INVALID_ARGUMENT


def test_device_error_bits_match_the_header():
    text = open(HEADER).read()
    assert re.search(r"#define LQ_DEVERR_WAIT_TIMEOUT 1u", text)
    assert re.search(r"#define LQ_DEVERR_BAD_POSITION 2u", text)
    assert re.search(r"#define LQ_POS_PER_SEQUENCE \(-1\)", text)
    assert (lq.LQ_DEVERR_WAIT_TIMEOUT, lq.LQ_DEVERR_BAD_POSITION, lq.LQ_POS_PER_SEQUENCE) == (1, 2, -1)


# --------------------------------------------------------------------------
# The Python binding checks every tensor before calling the library
# --------------------------------------------------------------------------

@pytest.fixture
def no_library(monkeypatch):
    """Any call that reaches the library fails the test."""
    def _refuse(*a, **k):
        raise AssertionError("the library was called")
    monkeypatch.setattr(lq, "load_library", _refuse)


def _cpu_tokens(cfg, n, io=None):
    import torch
    io = io or cfg.io_torch_dtype
    B, H = cfg.batch, cfg.heads
    return dict(q=torch.zeros((B, n, H, cfg.d_k), dtype=io), k=torch.zeros((B, n, H, cfg.d_k), dtype=io),
                v=torch.zeros((B, n, H, cfg.d_v), dtype=io),
                alpha=torch.ones((B, n, H, cfg.gdim) if cfg.gdim > 1 else (B, n, H)),
                beta=torch.ones((B, n, H)), o=torch.zeros((B, n, H, cfg.d_v), dtype=io))


def test_binding_rejects_bad_tensors_before_the_library(no_library):
    import torch
    cfg = lq.Config(batch=2, heads=3, d_k=64, d_v=128, window=4, n_comp=2, gate=lq.LQ_GATE_DIAG)
    st = lq.State(cfg, "cpu")
    t = _cpu_tokens(cfg, 2)
    # wrong io dtype
    bad = dict(t, q=t["q"].float())
    with pytest.raises(TypeError, match="q: dtype"):
        lq.lq_decode_window(st, bad["q"], bad["k"], bad["v"], bad["alpha"], bad["beta"], 2, bad["o"])
    # one token short for n_steps = 2
    bad = dict(t, v=t["v"][:, :1].contiguous())
    with pytest.raises(ValueError, match="v: .* elements"):
        lq.lq_decode_window(st, bad["q"], bad["k"], bad["v"], bad["alpha"], bad["beta"], 2, bad["o"])
    # a scalar gate's alpha for a diagonal-gate configuration
    bad = dict(t, alpha=torch.ones((2, 2, 3)))
    with pytest.raises(ValueError, match="alpha"):
        lq.lq_decode_window(st, bad["q"], bad["k"], bad["v"], bad["alpha"], bad["beta"], 2, bad["o"])
    # non-contiguous
    bad = dict(t, k=torch.zeros((2, 3, 2, 64), dtype=cfg.io_torch_dtype).transpose(1, 2))
    with pytest.raises(ValueError, match="k: not contiguous"):
        lq.lq_decode_window(st, bad["q"], bad["k"], bad["v"], bad["alpha"], bad["beta"], 2, bad["o"])
    # right sizes, but host memory
    with pytest.raises(ValueError, match="CUDA"):
        lq.lq_decode_window(st, t["q"], t["k"], t["v"], t["alpha"], t["beta"], 2, t["o"])
    # per-sequence positions: int32 [B]
    t1 = _cpu_tokens(cfg, 1)
    with pytest.raises(TypeError, match="seq_pos"):
        lq.lq_decode_ragged(st, torch.zeros(2, dtype=torch.int64), *[t1[x] for x in
                            ("q", "k", "v", "alpha", "beta", "o")])
    with pytest.raises(ValueError, match="seq_pos"):
        lq.lq_ragged_flush(st, torch.zeros(3, dtype=torch.int32))
    # snapshots must match the configuration
    other = lq.Snapshot(lq.Config(batch=2, heads=3, d_k=64, d_v=64, window=4, n_comp=2), "cpu")
    with pytest.raises(ValueError, match="dst.codes"):
        lq.lq_state_snapshot(st, other)
    with pytest.raises(ValueError, match="src.codes"):
        lq.lq_state_restore(st, other)
    # init: the FP32 state's size
    with pytest.raises(ValueError, match="S_init"):
        lq.lq_state_init(st, torch.zeros((6, 128, 63)))
    # prefill: state size, snapshot count
    tp = _cpu_tokens(cfg, 128)
    S = torch.zeros((6, 128, 64))
    with pytest.raises(ValueError, match="S_fp32"):
        lq.lq_prefill_chunk(st, S[:5], tp["q"], tp["k"], tp["v"], tp["alpha"], tp["beta"], 128, 64,
                            None, tp["o"])
    with pytest.raises(ValueError, match="snaps"):
        lq.lq_prefill_chunk(st, S, tp["q"], tp["k"], tp["v"], tp["alpha"], tp["beta"], 128, 64,
                            [lq.Snapshot(cfg, "cpu")], tp["o"])
    # the FP32 comparator: bf16 state
    with pytest.raises(TypeError, match="S: dtype"):
        lq.lq_fp32_step(cfg, S.bfloat16(), t1["q"], t1["k"], t1["v"], t1["alpha"], t1["beta"], 1,
                        t1["o"])


def test_prefill_workspace_bytes():
    """Two passes (one prepared while the other is scanned) of 16 chunks of
    64 tokens, 48 KB ([PT; T], 128 x 64 values in three BF16 parts) per chunk
    and head; 0 where the tensor-core prefill does not apply."""
    cfg = lq.Config(batch=2, heads=32, d_k=128, d_v=128, io_dtype=lq.LQ_BF16)
    assert lq.lq_prefill_workspace_bytes(cfg) == 2 * 16 * 64 * 49152
    cfg.d_v = 64
    assert lq.lq_prefill_workspace_bytes(cfg) == 2 * 16 * 64 * 49152
    for field, val in (("io_dtype", lq.LQ_F32), ("gate", lq.LQ_GATE_DIAG), ("d_k", 64)):
        c2 = lq.Config(batch=2, heads=32, d_k=128, d_v=128, io_dtype=lq.LQ_BF16)
        setattr(c2, field, val)
        assert lq.lq_prefill_workspace_bytes(c2) == 0, field
    cfg.window = 0
    assert lq.lq_prefill_workspace_bytes(cfg) == -1
