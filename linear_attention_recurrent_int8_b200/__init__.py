"""Python binding of liblq (include/lq.h): int8 per-window recurrent-state
decode for delta-rule linear attention on NVIDIA B200.

This module only marshals arguments: torch tensors become device pointers,
torch streams become ``cudaStream_t``.  Every step of the computation runs in
the CUDA kernels of ``liblq.so``; there is no CPU or PyTorch fallback, and a
missing or unloadable library raises.

The functions carry the C names (``lq_state_init``, ``lq_decode_window``,
``lq_window_commit``, ``lq_prefill_chunk``, ``lq_state_snapshot``,
``lq_state_restore``, ``lq_fp32_step``, ...).  ``State`` and ``Snapshot`` own
the torch tensors whose pointers the C structs hold.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblq.so")

LQ_OK, LQ_ERR_INVALID_ARGUMENT, LQ_ERR_UNSUPPORTED, LQ_ERR_WINDOW_FULL, \
    LQ_ERR_WINDOW_OPEN, LQ_ERR_MISALIGNED, LQ_ERR_CUDA = range(7)
LQ_GATE_SCALAR, LQ_GATE_DIAG = 0, 1
LQ_F32, LQ_BF16 = 0, 1
LQ_COMP_ROWS, LQ_COMP_SVD = 0, 1
LQ_POS_PER_SEQUENCE = -1
LQ_DEVERR_WAIT_TIMEOUT, LQ_DEVERR_BAD_POSITION = 1, 2

# Every symbol include/lq.h declares.
ABI_SYMBOLS = ("lq_buffer_elems", "lq_state_init", "lq_decode_window", "lq_decode_ragged",
               "lq_ragged_flush", "lq_window_commit",
               "lq_prefill_chunk", "lq_prefill_chunk_noalloc", "lq_prefill_workspace_bytes", "lq_state_snapshot", "lq_state_restore", "lq_fp32_step",
               "lq_state_destroy", "lq_status_string", "lq_device_errors")


class LQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_name(status)}")
        self.status = status


class LqConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "heads", "d_k", "d_v", "window", "n_comp",
                                              "gate", "io_dtype", "smoothing", "auto_commit", "delta",
                                              "bits", "comp_rule")]


class LqSnapshot(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("row_scale", ctypes.c_void_p),
                ("col_smooth", ctypes.c_void_p), ("comp_row", ctypes.c_void_p),
                ("comp_val", ctypes.c_void_p), ("comp_u", ctypes.c_void_p)]


class LqState(ctypes.Structure):
    _fields_ = [("cfg", LqConfig), ("snap", LqSnapshot), ("buf_gate", ctypes.c_void_p),
                ("buf_k", ctypes.c_void_p), ("buf_u", ctypes.c_void_p), ("pos", ctypes.c_int32),
                ("impl", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def load_library(build: bool = True):
    """Loads liblq.so, compiling it first when it is missing or stale."""
    global _lib
    with _lock:
        if _lib is None:
            if build:
                from .build import build_library
                build_library()
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"liblq.so not found at {LIB_PATH}")
            lib = ctypes.CDLL(LIB_PATH)
            P, I32 = ctypes.c_void_p, ctypes.c_int32
            sig = {
                "lq_buffer_elems": (ctypes.c_int64, [ctypes.POINTER(LqConfig), I32]),
                "lq_state_init": (I32, [ctypes.POINTER(LqState), ctypes.POINTER(LqConfig), P, P]),
                "lq_decode_window": (I32, [ctypes.POINTER(LqState), P, P, P, P, P, I32, P, P]),
                "lq_decode_ragged": (I32, [ctypes.POINTER(LqState), P, P, P, P, P, P, P, P]),
                "lq_ragged_flush": (I32, [ctypes.POINTER(LqState), P, P]),
                "lq_window_commit": (I32, [ctypes.POINTER(LqState), P]),
                "lq_prefill_chunk": (I32, [ctypes.POINTER(LqState), P, P, P, P, P, P, I32, I32,
                                           ctypes.POINTER(LqSnapshot), P, P, ctypes.c_size_t, P]),
                "lq_prefill_workspace_bytes": (ctypes.c_int64, [ctypes.POINTER(LqConfig)]),
                "lq_prefill_chunk_noalloc": (I32, [ctypes.POINTER(LqState), P, P, P, P, P, P, I32,
                                                   I32, ctypes.POINTER(LqSnapshot), P, P]),
                "lq_state_snapshot": (I32, [ctypes.POINTER(LqState), ctypes.POINTER(LqSnapshot), P]),
                "lq_state_restore": (I32, [ctypes.POINTER(LqState), ctypes.POINTER(LqSnapshot), P]),
                "lq_fp32_step": (I32, [ctypes.POINTER(LqConfig), P, P, P, P, P, P, I32, P, P]),
                "lq_state_destroy": (None, [ctypes.POINTER(LqState)]),
                "lq_status_string": (ctypes.c_char_p, [I32]),
                "lq_device_errors": (I32, [ctypes.POINTER(ctypes.c_uint32)]),
            }
            for name, (res, args) in sig.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def status_name(status: int) -> str:
    return lq_status_string(status)


def _check(status: int, where: str):
    if status != LQ_OK:
        raise LQError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# --------------------------------------------------------------------------
# Argument checks (before any call into the library)
# --------------------------------------------------------------------------
#
# The library checks pointers, sizes and alignment, but a pointer carries no
# length: a tensor that is too small, of the wrong dtype or on another device
# would be read past its end by the kernels' bulk copies.  Every wrapper
# therefore checks each tensor against the configuration first -- dtype,
# exact element count, contiguity, then that it lives on the state's CUDA
# device -- and raises before the library is called.

def _check_layout(t, name: str, dtype, numel: int, optional: bool = False) -> bool:
    """dtype, element count and contiguity; False for an absent optional tensor."""
    import torch
    if t is None:
        if optional:
            return False
        raise ValueError(f"{name}: a tensor is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel} (shape {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name}: not contiguous")
    return True


def _check_device(t, name: str, device):
    import torch
    dev = torch.device(device)
    if t.device.type != "cuda" or dev.type != "cuda":
        raise ValueError(f"{name}: on {t.device}, expected a CUDA tensor on {dev}")
    if dev.index is not None and t.device.index != dev.index:
        raise ValueError(f"{name}: on {t.device}, expected {dev}")


def _check_tensors(device, *specs):
    """specs: (tensor, name, dtype, numel[, optional]).  Every tensor's layout
    is checked first, then every present tensor's device."""
    present = [sp for sp in specs if _check_layout(*sp)]
    for sp in present:
        _check_device(sp[0], sp[1], device)


def _token_specs(cfg: "Config", n: int, q, k, v, alpha, beta, o):
    import torch
    B, H = cfg.batch, cfg.heads
    io = cfg.io_torch_dtype
    return [(q, "q", io, B * n * H * cfg.d_k), (k, "k", io, B * n * H * cfg.d_k),
            (v, "v", io, B * n * H * cfg.d_v),
            (alpha, "alpha", torch.float32, B * n * H * cfg.gdim),
            (beta, "beta", torch.float32, B * n * H), (o, "o", io, B * n * H * cfg.d_v)]


def _snapshot_specs(cfg: "Config", snap: "Snapshot", name: str):
    import torch
    bh = cfg.batch * cfg.heads
    t = snap.t
    specs = [(t["codes"], f"{name}.codes", cfg.code_torch_dtype, bh * cfg.d_v * cfg.code_cols),
             (t["row_scale"], f"{name}.row_scale", torch.float32, bh * cfg.d_v),
             (t["col_smooth"], f"{name}.col_smooth", torch.float32, bh * cfg.d_k)]
    if cfg.n_comp > 0:
        specs += [(t["comp_row"], f"{name}.comp_row", torch.int32, bh * cfg.n_comp),
                  (t["comp_val"], f"{name}.comp_val", torch.float32, bh * cfg.n_comp * cfg.d_k)]
    if cfg.svd:
        specs += [(t["comp_u"], f"{name}.comp_u", torch.float32, bh * cfg.n_comp * cfg.d_v)]
    return specs


# --------------------------------------------------------------------------
# Configuration, snapshot and state holders
# --------------------------------------------------------------------------

@dataclass
class Config:
    batch: int
    heads: int
    d_k: int = 128
    d_v: int = 128
    window: int = 16
    n_comp: int = 4
    gate: int = LQ_GATE_SCALAR
    io_dtype: int = LQ_BF16
    smoothing: int = 1
    auto_commit: int = 1
    delta: int = 1
    bits: int = 8  # code width: 8, 6 (one code per byte), 4 (two per byte), 16 (BF16 residual)
    comp_rule: int = LQ_COMP_ROWS  # LQ_COMP_ROWS (top-r rows) or LQ_COMP_SVD (top-r singular triplets)

    def c(self) -> LqConfig:
        return LqConfig(self.batch, self.heads, self.d_k, self.d_v, self.window, self.n_comp,
                        self.gate, self.io_dtype, self.smoothing, self.auto_commit, self.delta,
                        self.bits, self.comp_rule)

    @property
    def svd(self) -> bool:
        """The SVD compensator rule is in effect (with r = 0 the rules coincide)."""
        return self.comp_rule == LQ_COMP_SVD and self.n_comp > 0

    @property
    def code_cols(self) -> int:
        """Elements of one value row of the residual (d_k, or d_k / 2 bytes at 4 bits)."""
        return self.d_k // 2 if self.bits == 4 else self.d_k

    @property
    def code_torch_dtype(self):
        import torch
        return {4: torch.uint8, 16: torch.bfloat16}.get(self.bits, torch.int8)

    @property
    def gdim(self) -> int:
        return self.d_k if self.gate == LQ_GATE_DIAG else 1

    @property
    def io_torch_dtype(self):
        import torch
        return torch.bfloat16 if self.io_dtype == LQ_BF16 else torch.float32


class Snapshot:
    """Device tensors of one quantized boundary state (layouts of lq_snapshot)."""

    def __init__(self, cfg: Config, device, tensors: dict | None = None):
        import torch
        bh = cfg.batch * cfg.heads
        if tensors is None:
            tensors = dict(
                codes=torch.zeros((bh, cfg.d_v, cfg.code_cols), dtype=cfg.code_torch_dtype,
                                  device=device),
                row_scale=torch.zeros((bh, cfg.d_v), dtype=torch.float32, device=device),
                col_smooth=torch.ones((bh, cfg.d_k), dtype=torch.float32, device=device),
                comp_row=torch.zeros((bh, cfg.n_comp), dtype=torch.int32, device=device),
                comp_val=torch.zeros((bh, cfg.n_comp, cfg.d_k), dtype=torch.float32, device=device),
            )
            if cfg.svd:
                tensors["comp_u"] = torch.zeros((bh, cfg.n_comp, cfg.d_v), dtype=torch.float32,
                                                device=device)
        self.t = tensors

    def __getitem__(self, key):
        return self.t[key]

    def c(self) -> LqSnapshot:
        t = self.t
        has = t["comp_row"].numel() > 0
        cu = t.get("comp_u")
        return LqSnapshot(t["codes"].data_ptr(), t["row_scale"].data_ptr(),
                          t["col_smooth"].data_ptr(),
                          t["comp_row"].data_ptr() if has else None,
                          t["comp_val"].data_ptr() if has else None,
                          cu.data_ptr() if cu is not None and cu.numel() > 0 else None)

    def cpu(self) -> dict:
        return {k: v.cpu().numpy() for k, v in self.t.items()}


class State:
    """A decode state: the boundary snapshot plus the window buffers, all
    device memory allocated here by torch, and the C struct pointing at them."""

    def __init__(self, cfg: Config, device="cuda"):
        import torch
        self.cfg = cfg
        self.device = torch.device(device)
        bh = cfg.batch * cfg.heads
        self.snap = Snapshot(cfg, self.device)
        self.buf_gate = torch.zeros((bh, cfg.window, cfg.gdim), dtype=torch.float32, device=device)
        self.buf_k = torch.zeros((bh, cfg.window, cfg.d_k), dtype=torch.float32, device=device)
        self.buf_u = torch.zeros((bh, cfg.window, cfg.d_v), dtype=torch.float32, device=device)
        self.c = LqState()
        self.c.cfg = cfg.c()
        self.c.snap = self.snap.c()
        self.c.buf_gate = self.buf_gate.data_ptr()
        self.c.buf_k = self.buf_k.data_ptr()
        self.c.buf_u = self.buf_u.data_ptr()
        self.c.pos = 0
        self.c.impl = None

    @property
    def pos(self) -> int:
        return self.c.pos


# --------------------------------------------------------------------------
# The C entry points, same names
# --------------------------------------------------------------------------

def lq_status_string(status: int) -> str:
    return load_library().lq_status_string(int(status)).decode()


def lq_buffer_elems(cfg: Config, which: int) -> int:
    c = cfg.c()
    return load_library().lq_buffer_elems(ctypes.byref(c), which)


def lq_state_init(st: State, S_init=None, stream=None) -> None:
    import torch
    cfg = st.cfg
    _check_tensors(st.device, (S_init, "S_init", torch.float32,
                               cfg.batch * cfg.heads * cfg.d_v * cfg.d_k, True),
                   *_snapshot_specs(cfg, st.snap, "state.snap"))
    c = st.cfg.c()
    _check(load_library().lq_state_init(ctypes.byref(st.c), ctypes.byref(c), _ptr(S_init),
                                        _stream(stream)), "lq_state_init")


def lq_decode_window(st: State, q, k, v, alpha, beta, n_steps: int, o, stream=None) -> None:
    if int(n_steps) > 0:
        _check_tensors(st.device, *_token_specs(st.cfg, int(n_steps), q, k, v, alpha, beta, o))
    _check(load_library().lq_decode_window(ctypes.byref(st.c), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(alpha), _ptr(beta), int(n_steps), _ptr(o),
                                           _stream(stream)), "lq_decode_window")


def lq_decode_ragged(st: State, seq_pos, q, k, v, alpha, beta, o, stream=None) -> None:
    """One token per active sequence at its own window position (seq_pos:
    int32 device tensor [B], negative = idle slot; updated in place)."""
    import torch
    _check_tensors(st.device, (seq_pos, "seq_pos", torch.int32, st.cfg.batch),
                   *_token_specs(st.cfg, 1, q, k, v, alpha, beta, o))
    _check(load_library().lq_decode_ragged(ctypes.byref(st.c), _ptr(seq_pos), _ptr(q), _ptr(k),
                                           _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                           _stream(stream)), "lq_decode_ragged")


def lq_ragged_flush(st: State, seq_pos, stream=None) -> None:
    """Commits every sequence's open window (1 <= seq_pos[b] < W) and sets
    those positions to 0; afterwards st.pos == 0."""
    import torch
    _check_tensors(st.device, (seq_pos, "seq_pos", torch.int32, st.cfg.batch))
    _check(load_library().lq_ragged_flush(ctypes.byref(st.c), _ptr(seq_pos), _stream(stream)),
           "lq_ragged_flush")


def lq_window_commit(st: State, stream=None) -> None:
    _check(load_library().lq_window_commit(ctypes.byref(st.c), _stream(stream)), "lq_window_commit")


def lq_prefill_workspace_bytes(cfg: Config) -> int:
    c = cfg.c()
    return load_library().lq_prefill_workspace_bytes(ctypes.byref(c))


def lq_prefill_chunk(st: State, S_fp32, q, k, v, alpha, beta, T: int, snapshot_every: int,
                     snaps, o, stream=None, workspace="auto") -> None:
    """workspace: "auto" allocates (torch) the size lq_prefill_workspace_bytes
    gives for this call; a CUDA tensor is used as it is; None runs the
    prefill token by token."""
    import torch
    cfg = st.cfg
    if int(T) > 0:
        specs = [(S_fp32, "S_fp32", torch.float32, cfg.batch * cfg.heads * cfg.d_v * cfg.d_k)]
        specs += _token_specs(cfg, int(T), q, k, v, alpha, beta, o)
        if snaps is not None:
            if int(snapshot_every) < 1 or int(T) % int(snapshot_every) != 0 or \
                    len(snaps) != int(T) // int(snapshot_every):
                raise ValueError(f"snaps: {len(snaps)} snapshots for T = {T}, "
                                 f"snapshot_every = {snapshot_every}")
            for i, sn in enumerate(snaps):
                specs += _snapshot_specs(cfg, sn, f"snaps[{i}]")
        _check_tensors(st.device, *specs)
    ws, ws_bytes = None, 0
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace: {workspace!r}")
        n = lq_prefill_workspace_bytes(cfg) if int(T) > 0 else 0
        if n > 0:
            ws = torch.empty(n, dtype=torch.uint8, device=st.device)
    elif workspace is not None:
        if not isinstance(workspace, torch.Tensor) or not workspace.is_contiguous():
            raise ValueError("workspace: expected a contiguous tensor")
        _check_device(workspace, "workspace", st.device)
        ws = workspace
    if ws is not None:
        ws_bytes = ws.numel() * ws.element_size()
    arr = None
    if snaps is not None:
        arr = (LqSnapshot * len(snaps))(*[s.c() for s in snaps])
    _check(load_library().lq_prefill_chunk(ctypes.byref(st.c), _ptr(S_fp32), _ptr(q), _ptr(k),
                                           _ptr(v), _ptr(alpha), _ptr(beta), int(T),
                                           int(snapshot_every), arr, _ptr(o), _ptr(ws), ws_bytes,
                                           _stream(stream)),
           "lq_prefill_chunk")


def lq_prefill_chunk_noalloc(st: State, S_fp32, q, k, v, alpha, beta, T: int,
                             snapshot_every: int, snaps, o, stream=None) -> None:
    """lq_prefill_chunk with the library's fixed scratch array instead of a
    workspace: for callers that cannot hand out more device memory.  Neither
    this wrapper nor the library allocates anything."""
    import torch
    cfg = st.cfg
    if int(T) > 0:
        specs = [(S_fp32, "S_fp32", torch.float32, cfg.batch * cfg.heads * cfg.d_v * cfg.d_k)]
        specs += _token_specs(cfg, int(T), q, k, v, alpha, beta, o)
        if snaps is not None:
            if int(snapshot_every) < 1 or int(T) % int(snapshot_every) != 0 or \
                    len(snaps) != int(T) // int(snapshot_every):
                raise ValueError(f"snaps: {len(snaps)} snapshots for T = {T}, "
                                 f"snapshot_every = {snapshot_every}")
            for i, sn in enumerate(snaps):
                specs += _snapshot_specs(cfg, sn, f"snaps[{i}]")
        _check_tensors(st.device, *specs)
    arr = None
    if snaps is not None:
        arr = (LqSnapshot * len(snaps))(*[s.c() for s in snaps])
    _check(load_library().lq_prefill_chunk_noalloc(ctypes.byref(st.c), _ptr(S_fp32), _ptr(q), _ptr(k),
                                                   _ptr(v), _ptr(alpha), _ptr(beta), int(T),
                                                   int(snapshot_every), arr, _ptr(o), _stream(stream)),
           "lq_prefill_chunk_noalloc")


def lq_state_snapshot(st: State, dst: Snapshot, stream=None) -> None:
    _check_tensors(st.device, *_snapshot_specs(st.cfg, dst, "dst"))
    c = dst.c()
    _check(load_library().lq_state_snapshot(ctypes.byref(st.c), ctypes.byref(c), _stream(stream)),
           "lq_state_snapshot")


def lq_state_restore(st: State, src: Snapshot, stream=None) -> None:
    _check_tensors(st.device, *_snapshot_specs(st.cfg, src, "src"))
    c = src.c()
    _check(load_library().lq_state_restore(ctypes.byref(st.c), ctypes.byref(c), _stream(stream)),
           "lq_state_restore")


def lq_fp32_step(cfg: Config, S, q, k, v, alpha, beta, n_steps: int, o, stream=None) -> None:
    import torch
    if int(n_steps) > 0:
        dev = S.device if isinstance(S, torch.Tensor) else "cuda"
        _check_tensors(dev, (S, "S", torch.float32, cfg.batch * cfg.heads * cfg.d_v * cfg.d_k),
                       *_token_specs(cfg, int(n_steps), q, k, v, alpha, beta, o))
    c = cfg.c()
    _check(load_library().lq_fp32_step(ctypes.byref(c), _ptr(S), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(alpha), _ptr(beta), int(n_steps), _ptr(o),
                                       _stream(stream)), "lq_fp32_step")


def lq_state_destroy(st: State) -> None:
    load_library().lq_state_destroy(ctypes.byref(st.c))


def lq_device_errors() -> int:
    flags = ctypes.c_uint32(0)
    _check(load_library().lq_device_errors(ctypes.byref(flags)), "lq_device_errors")
    return flags.value
