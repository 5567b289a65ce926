"""Python binding of the Lighthouse C ABI (include/lh.h).

Argument marshalling only: every stage runs in liblh.so's CUDA kernels.
PyTorch provides device memory and the current stream.  Importing this module
loads liblh.so and fails loudly if it is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# LH_LIBRARY selects another build of the library (for example a variant
# compiled with different tile constants); the default is the in-tree one.
LIB_PATH = os.environ.get("LH_LIBRARY") or os.path.join(HERE, "liblh.so")

LH_OK, LH_ERR_INVALID_ARG, LH_ERR_UNSUPPORTED, LH_ERR_WORKSPACE, LH_ERR_CUDA, LH_ERR_TIMEOUT = range(6)
LH_F32, LH_BF16 = 0, 1
MAX_LEVELS = 8
DTYPES = {"f32": LH_F32, "bf16": LH_BF16}
TORCH_DTYPE = {LH_F32: torch.float32, LH_BF16: torch.bfloat16}

# Every exported name declared in include/lh.h.
EXPORTS = (
    "lh_plan_init", "lh_pyramid", "lh_score", "lh_pyramid_score", "lh_topk", "lh_gather",
    "lh_attn_fwd", "lh_attn_bwd_ws_bytes", "lh_attn_bwd", "lh_scatter", "lh_scatter_bwd",
    "lh_gather_bwd", "lh_forward", "lh_backward", "lh_device_status", "lh_status_string",
    "lh_last_error", "lh_plan_bytes", "lh_attn_bwd_static", "lh_set_deterministic",
    "lh_selftest_wait_timeout",
)


SELECT = {"joint": 0, "descent": 1, "regional": 2}


class LhConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "N", "d", "p", "L", "k", "dtype", "select")]


_I64 = ctypes.c_int64


class LhPlan(ctypes.Structure):
    _fields_ = [
        ("c", LhConfig),
        ("P", _I64 * MAX_LEVELS),
        ("n", _I64 * MAX_LEVELS),
        ("flat_off", _I64 * (MAX_LEVELS + 1)),
        ("pyr_off", _I64 * MAX_LEVELS),
    ] + [(n, _I64) for n in (
        "Ntot", "Npyr", "M", "Ksel", "S", "elem_bytes",
        "ctx_bytes", "ws_bytes", "topk_ws_bytes", "attn_bwd_ws_bytes",
        "ctx_sel_idx", "ctx_slot_of", "ctx_Qg", "ctx_Kg", "ctx_Vg", "ctx_Og", "ctx_lse",
        "ws_pyrQ", "ws_pyrK", "ws_pyrV", "ws_scores", "ws_topk",
        "ws_dOg", "ws_D", "ws_dQg", "ws_dKg", "ws_dVg", "ws_attn")]


class LighthouseError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({detail})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m long_context_hierarchical_b200.build`"
            " (the Lighthouse layer has no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    PLAN = ctypes.POINTER(LhPlan)
    sig = {
        "lh_plan_init": (ctypes.POINTER(LhConfig), PLAN),
        "lh_pyramid": (PLAN, P, P, P, P, P, P, P),
        "lh_score": (PLAN, P, P, P, P),
        "lh_pyramid_score": (PLAN, P, P, P, P, P, P, P, P),
        "lh_topk": (PLAN, P, P, P, P, SZ, P),
        "lh_gather": (PLAN, P, P, P, P, P, P, P, P, P, P, P),
        "lh_attn_fwd": (I64, I64, I32, I32, P, P, P, P, P, P),
        "lh_attn_bwd": (I64, I64, I32, I32, P, P, P, P, P, P, P, P, P, P, P, SZ, P),
        "lh_scatter": (PLAN, P, P, P, P),
        "lh_scatter_bwd": (PLAN, P, P, P, P, P, P),
        "lh_gather_bwd": (PLAN, P, P, P, P, P, P, P, P),
        "lh_forward": (PLAN, P, P, P, P, P, SZ, P, SZ, P),
        "lh_backward": (PLAN, P, P, SZ, P, P, P, P, SZ, P),
        "lh_device_status": (ctypes.c_int,),
        "lh_selftest_wait_timeout": (P,),
        "lh_attn_bwd_static": (I64, I64, I32, I32, P, P, P, P, P, P, P, P, P, P),
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = list(args)
        f.restype = ctypes.c_int
    lib.lh_attn_bwd_ws_bytes.argtypes = [I64, I64, I32, I32]
    lib.lh_attn_bwd_ws_bytes.restype = I64
    lib.lh_status_string.argtypes = [ctypes.c_int]
    lib.lh_status_string.restype = ctypes.c_char_p
    lib.lh_last_error.argtypes = []
    lib.lh_last_error.restype = ctypes.c_char_p
    lib.lh_plan_bytes.argtypes = []
    lib.lh_plan_bytes.restype = I64
    lib.lh_set_deterministic.argtypes = [ctypes.c_int]
    lib.lh_set_deterministic.restype = None
    if lib.lh_plan_bytes() != ctypes.sizeof(LhPlan):
        raise ImportError("lh_plan layout of liblh.so does not match this binding")
    return lib


LIB = _load()


def _check(status: int, where: str):
    if status != LH_OK:
        detail = (LIB.lh_last_error() or b"").decode() or LIB.lh_status_string(status).decode()
        raise LighthouseError(status, where, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(t, name: str, dtype, numel: int):
    """Check a tensor the library will read or write as ``numel`` contiguous
    elements of ``dtype`` in device memory (the C ABI sees only its pointer)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the call needs {numel}")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor (got {t.device})")


def _require_tokens(pl, **tensors):
    """[B,H,N,d] tensors of the plan's dtype."""
    c = pl.raw.c
    for name, t in tensors.items():
        _require(t, name, pl.dtype, c.B * c.H * c.N * c.d)


def _require_rows(pl, **tensors):
    """[B,H,S,d] gathered tensors of the plan's dtype."""
    c = pl.raw.c
    for name, t in tensors.items():
        _require(t, name, pl.dtype, c.B * c.H * pl.S * c.d)


def _attn_shape(Qg, **others):
    """(BH, S, d) of [..., S, d] attention operands; every other operand has
    Qg's dtype and size."""
    if not isinstance(Qg, torch.Tensor) or Qg.dim() < 2:
        raise ValueError("Qg: expected a tensor of shape [..., S, d]")
    if Qg.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"Qg: dtype {Qg.dtype}, expected torch.bfloat16 or torch.float32")
    S, d = Qg.shape[-2], Qg.shape[-1]
    _require(Qg, "Qg", Qg.dtype, Qg.numel())
    for name, t in others.items():
        _require(t, name, Qg.dtype, Qg.numel())
    return Qg.numel() // max(S * d, 1), S, d


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Plan:
    """Sizes and buffer layout of one layer configuration (from lh_plan_init)."""
    raw: LhPlan

    @property
    def S(self):
        return self.raw.S

    @property
    def M(self):
        return self.raw.M

    @property
    def Ntot(self):
        return self.raw.Ntot

    @property
    def Npyr(self):
        return self.raw.Npyr

    @property
    def Ksel(self):
        return self.raw.Ksel

    @property
    def BH(self):
        return self.raw.c.B * self.raw.c.H

    @property
    def dtype(self):
        return TORCH_DTYPE[self.raw.c.dtype]

    def byref(self):
        return ctypes.byref(self.raw)


def plan(B: int, H: int, N: int, d: int = 64, p: int = 4, L: int = 3, k: int = 0,
         dtype: str = "bf16", select: str = "joint") -> Plan:
    """select: "joint" (one top-K over all candidate levels), "descent"
    (hierarchical descent from the coarsest level) or "regional" (every
    2048-candidate region keeps its share of the budget)."""
    cfg = LhConfig(B, H, N, d, p, L, k, DTYPES[dtype], SELECT[select])
    raw = LhPlan()
    _check(LIB.lh_plan_init(ctypes.byref(cfg), ctypes.byref(raw)), "lh_plan_init")
    return Plan(raw)


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def _bytes(n, device):
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


# --- stages -----------------------------------------------------------------


def pyramid_score(pl: Plan, Q, K, V, stream=None):
    """Levels 1..L-1 of Q, K, V ([B,H,Npyr,d] each) and candidate scores [B,H,M]."""
    _require_tokens(pl, Q=Q, K=K, V=V)
    c = pl.raw.c
    dev = Q.device
    pyr = [_empty((c.B, c.H, max(pl.Npyr, 1), c.d), Q.dtype, dev) for _ in range(3)]
    scores = _empty((c.B, c.H, max(pl.M, 1)), torch.float32, dev)
    _check(LIB.lh_pyramid_score(pl.byref(), _ptr(Q), _ptr(K), _ptr(V), *map(_ptr, pyr),
                                _ptr(scores), _stream(stream)), "lh_pyramid_score")
    return pyr, scores


def pyramid(pl: Plan, Q, K, V, stream=None):
    _require_tokens(pl, Q=Q, K=K, V=V)
    c = pl.raw.c
    pyr = [_empty((c.B, c.H, max(pl.Npyr, 1), c.d), Q.dtype, Q.device) for _ in range(3)]
    _check(LIB.lh_pyramid(pl.byref(), _ptr(Q), _ptr(K), _ptr(V), *map(_ptr, pyr),
                          _stream(stream)), "lh_pyramid")
    return pyr


def score(pl: Plan, Q, K, stream=None):
    _require_tokens(pl, Q=Q, K=K)
    c = pl.raw.c
    scores = _empty((c.B, c.H, max(pl.M, 1)), torch.float32, Q.device)
    _check(LIB.lh_score(pl.byref(), _ptr(Q), _ptr(K), _ptr(scores), _stream(stream)), "lh_score")
    return scores


def topk(pl: Plan, scores, stream=None):
    """(sel_idx [B,H,S] int32, slot_of [B,H,Ntot] int32) from scores [B,H,M]."""
    c = pl.raw.c
    _require(scores, "scores", torch.float32, c.B * c.H * pl.M)
    dev = scores.device
    sel = _empty((c.B, c.H, pl.S), torch.int32, dev)
    inv = _empty((c.B, c.H, pl.Ntot), torch.int32, dev)
    ws = _bytes(pl.raw.topk_ws_bytes, dev)
    _check(LIB.lh_topk(pl.byref(), _ptr(scores), _ptr(sel), _ptr(inv), _ptr(ws), ws.numel(),
                       _stream(stream)), "lh_topk")
    return sel, inv


def gather(pl: Plan, Q, K, V, pyr, sel_idx, stream=None):
    _require_tokens(pl, Q=Q, K=K, V=V)
    c = pl.raw.c
    if len(pyr) != 3:
        raise ValueError("pyr: expected the three pyramids (Q, K, V)")
    for name, t in zip(("pyrQ", "pyrK", "pyrV"), pyr):
        _require(t, name, pl.dtype, c.B * c.H * pl.Npyr * c.d)
    _require(sel_idx, "sel_idx", torch.int32, c.B * c.H * pl.S)
    out = [_empty((c.B, c.H, pl.S, c.d), Q.dtype, Q.device) for _ in range(3)]
    _check(LIB.lh_gather(pl.byref(), _ptr(Q), _ptr(K), _ptr(V), *map(_ptr, pyr), _ptr(sel_idx),
                         *map(_ptr, out), _stream(stream)), "lh_gather")
    return out


def _dtype_code(t):
    return LH_BF16 if t.dtype == torch.bfloat16 else LH_F32


def attn_fwd(Qg, Kg, Vg, stream=None):
    """Causal attention on [..., S, d] tensors: (O, lse[..., S] natural log)."""
    BH, S, d = _attn_shape(Qg, Kg=Kg, Vg=Vg)
    O = torch.empty_like(Qg)
    lse = _empty(Qg.shape[:-1], torch.float32, Qg.device)
    _check(LIB.lh_attn_fwd(BH, S, d, _dtype_code(Qg), _ptr(Qg), _ptr(Kg), _ptr(Vg), _ptr(O),
                           _ptr(lse), _stream(stream)), "lh_attn_fwd")
    return O, lse


def attn_bwd(Qg, Kg, Vg, Og, lse, dOg, D=None, stream=None):
    BH, S, d = _attn_shape(Qg, Kg=Kg, Vg=Vg, Og=Og, dOg=dOg)
    _require(lse, "lse", torch.float32, BH * S)
    if D is not None:
        _require(D, "D", torch.float32, BH * S)
    code = _dtype_code(Qg)
    dQ, dK, dV = torch.empty_like(Qg), torch.empty_like(Kg), torch.empty_like(Vg)
    ws = _bytes(LIB.lh_attn_bwd_ws_bytes(BH, S, d, code), Qg.device)
    _check(LIB.lh_attn_bwd(BH, S, d, code, _ptr(Qg), _ptr(Kg), _ptr(Vg), _ptr(Og), _ptr(lse),
                           _ptr(dOg), _ptr(D), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(ws), ws.numel(),
                           _stream(stream)), "lh_attn_bwd")
    return dQ, dK, dV


def attn_bwd_static(Qg, Kg, Vg, Og, lse, dOg, stream=None):
    """lh_attn_bwd with D computed into the library's own scratch array
    (no workspace: for callers that cannot allocate device memory)."""
    BH, S, d = _attn_shape(Qg, Kg=Kg, Vg=Vg, Og=Og, dOg=dOg)
    _require(lse, "lse", torch.float32, BH * S)
    dQ, dK, dV = torch.empty_like(Qg), torch.empty_like(Kg), torch.empty_like(Vg)
    _check(LIB.lh_attn_bwd_static(BH, S, d, _dtype_code(Qg), _ptr(Qg), _ptr(Kg), _ptr(Vg), _ptr(Og),
                                  _ptr(lse), _ptr(dOg), _ptr(dQ), _ptr(dK), _ptr(dV),
                                  _stream(stream)), "lh_attn_bwd_static")
    return dQ, dK, dV


def scatter(pl: Plan, Og, slot_of, stream=None):
    _require_rows(pl, Og=Og)
    c = pl.raw.c
    _require(slot_of, "slot_of", torch.int32, c.B * c.H * pl.Ntot)
    O = _empty((c.B, c.H, c.N, c.d), Og.dtype, Og.device)
    _check(LIB.lh_scatter(pl.byref(), _ptr(Og), _ptr(slot_of), _ptr(O), _stream(stream)),
           "lh_scatter")
    return O


def scatter_bwd(pl: Plan, dO, Og, sel_idx, stream=None):
    _require_tokens(pl, dO=dO)
    _require_rows(pl, Og=Og)
    c = pl.raw.c
    _require(sel_idx, "sel_idx", torch.int32, c.B * c.H * pl.S)
    dOg = _empty((c.B, c.H, pl.S, c.d), dO.dtype, dO.device)
    D = _empty((c.B, c.H, pl.S), torch.float32, dO.device)
    _check(LIB.lh_scatter_bwd(pl.byref(), _ptr(dO), _ptr(Og), _ptr(sel_idx), _ptr(dOg), _ptr(D),
                              _stream(stream)), "lh_scatter_bwd")
    return dOg, D


def gather_bwd(pl: Plan, dQg, dKg, dVg, slot_of, stream=None):
    _require_rows(pl, dQg=dQg, dKg=dKg, dVg=dVg)
    c = pl.raw.c
    _require(slot_of, "slot_of", torch.int32, c.B * c.H * pl.Ntot)
    out = [_empty((c.B, c.H, c.N, c.d), dQg.dtype, dQg.device) for _ in range(3)]
    _check(LIB.lh_gather_bwd(pl.byref(), _ptr(dQg), _ptr(dKg), _ptr(dVg), _ptr(slot_of),
                             *map(_ptr, out), _stream(stream)), "lh_gather_bwd")
    return out


# --- whole layer --------------------------------------------------------------


class Context:
    """The forward-to-backward buffer of one lh_forward call, with typed views."""

    def __init__(self, pl: Plan, device):
        self.plan = pl
        self.buf = _bytes(pl.raw.ctx_bytes, device)

    def _view(self, off, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return self.buf[off: off + nbytes].view(dtype).view(shape)

    @property
    def sel_idx(self):
        c = self.plan.raw.c
        return self._view(self.plan.raw.ctx_sel_idx, (c.B, c.H, self.plan.S), torch.int32)

    @property
    def slot_of(self):
        c = self.plan.raw.c
        return self._view(self.plan.raw.ctx_slot_of, (c.B, c.H, self.plan.Ntot), torch.int32)

    def gathered(self, name):
        c = self.plan.raw.c
        off = getattr(self.plan.raw, "ctx_" + name)
        return self._view(off, (c.B, c.H, self.plan.S, c.d), self.plan.dtype)

    @property
    def lse(self):
        c = self.plan.raw.c
        return self._view(self.plan.raw.ctx_lse, (c.B, c.H, self.plan.S), torch.float32)


class Workspace:
    def __init__(self, pl: Plan, device):
        self.buf = _bytes(pl.raw.ws_bytes, device)


def forward(pl: Plan, Q, K, V, O=None, ctx: Context | None = None, ws: Workspace | None = None,
            stream=None):
    """O = Lighthouse(Q, K, V); returns (O, ctx)."""
    _require_tokens(pl, Q=Q, K=K, V=V)
    dev = Q.device
    if O is None:
        O = torch.empty_like(Q)
    if ctx is None:
        ctx = Context(pl, dev)
    if ws is None:
        ws = Workspace(pl, dev)
    _require_tokens(pl, O=O)
    _require(ctx.buf, "ctx", torch.uint8, pl.raw.ctx_bytes)
    _require(ws.buf, "ws", torch.uint8, pl.raw.ws_bytes)
    _check(LIB.lh_forward(pl.byref(), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(ctx.buf),
                          ctx.buf.numel(), _ptr(ws.buf), ws.buf.numel(), _stream(stream)),
           "lh_forward")
    return O, ctx


def backward(pl: Plan, dO, ctx: Context, dQ=None, dK=None, dV=None, ws: Workspace | None = None,
             stream=None):
    """(dQ, dK, dV) from dO and the ctx of the matching forward."""
    _require_tokens(pl, dO=dO)
    if dQ is None:
        dQ, dK, dV = torch.empty_like(dO), torch.empty_like(dO), torch.empty_like(dO)
    if ws is None:
        ws = Workspace(pl, dO.device)
    _require_tokens(pl, dQ=dQ, dK=dK, dV=dV)
    _require(ctx.buf, "ctx", torch.uint8, pl.raw.ctx_bytes)
    _require(ws.buf, "ws", torch.uint8, pl.raw.ws_bytes)
    _check(LIB.lh_backward(pl.byref(), _ptr(dO), _ptr(ctx.buf), ctx.buf.numel(), _ptr(dQ),
                           _ptr(dK), _ptr(dV), _ptr(ws.buf), ws.buf.numel(), _stream(stream)),
           "lh_backward")
    return dQ, dK, dV


class HostPipeline:
    """Forward and backward of one layer per step on host (pinned) tensors.

    Each step copies Q, K, V, dO to the device, runs lh_forward and
    lh_backward, and copies O, dQ, dK, dV back.  Two device buffer sets and
    three streams let the copy-in of step i+1 and the copy-out of step i-1
    run while the kernels of step i do (PCIe is full duplex; the kernels use
    only the compute stream).  ``step`` enqueues and returns at once;
    ``synchronize`` waits for every enqueued step.  The host tensors passed to
    a step must stay untouched until it has completed.
    """

    def __init__(self, pl: Plan, device):
        c = pl.raw.c
        shape = (c.B, c.H, c.N, c.d)
        self.pl = pl
        self.inputs = [[torch.empty(shape, dtype=pl.dtype, device=device) for _ in range(4)]
                       for _ in range(2)]
        self.outputs = [[torch.empty(shape, dtype=pl.dtype, device=device) for _ in range(4)]
                        for _ in range(2)]
        self.ctx = Context(pl, device)
        self.ws = Workspace(pl, device)
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(device) for _ in range(3))
        self.copied_in = [torch.cuda.Event() for _ in range(2)]
        self.done = [torch.cuda.Event() for _ in range(2)]
        self.copied_out = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.n = 0

    def step(self, host_inputs, host_outputs):
        """host_inputs: (Q, K, V, dO); host_outputs: (O, dQ, dK, dV); pinned, [B,H,N,d]."""
        b = self.n % 2
        self.n += 1
        dev_in, dev_out = self.inputs[b], self.outputs[b]
        if self.used[b]:  # this buffer set's previous step has read its inputs
            self.s_in.wait_event(self.done[b])
        with torch.cuda.stream(self.s_in):
            for d, h in zip(dev_in, host_inputs):
                d.copy_(h, non_blocking=True)
            self.copied_in[b].record(self.s_in)
        self.s_run.wait_event(self.copied_in[b])
        if self.used[b]:  # and its outputs have left the device
            self.s_run.wait_event(self.copied_out[b])
        Q, K, V, dO = dev_in
        O, dQ, dK, dV = dev_out
        forward(self.pl, Q, K, V, O, self.ctx, self.ws, stream=self.s_run)
        backward(self.pl, dO, self.ctx, dQ, dK, dV, self.ws, stream=self.s_run)
        self.done[b].record(self.s_run)
        self.s_out.wait_event(self.done[b])
        with torch.cuda.stream(self.s_out):
            for h, d in zip(host_outputs, dev_out):
                h.copy_(d, non_blocking=True)
            self.copied_out[b].record(self.s_out)
        self.used[b] = True

    def wait_on(self, event):
        """Make every stream of the pipeline wait for `event` (e.g. a start marker)."""
        for st in (self.s_in, self.s_run, self.s_out):
            st.wait_event(event)

    def record_end(self, stream):
        """Make `stream` wait for everything enqueued so far."""
        for ev in self.copied_in + self.done + self.copied_out:
            stream.wait_event(ev)

    def synchronize(self):
        for st in (self.s_in, self.s_run, self.s_out):
            st.synchronize()


def set_deterministic(on: bool):
    """Process-wide: bit-reproducible bf16 attention backward (two kernels, no
    atomics) for lh_attn_bwd / lh_backward calls enqueued afterwards."""
    LIB.lh_set_deterministic(1 if on else 0)


def selftest_wait_timeout(stream=None):
    """Enqueue the failure-path self-test (a bounded wait that must give up);
    the next device_status() raises LighthouseError with LH_ERR_TIMEOUT."""
    _check(LIB.lh_selftest_wait_timeout(_stream(stream)), "lh_selftest_wait_timeout")


def device_status(reset: bool = True):
    _check(LIB.lh_device_status(1 if reset else 0), "lh_device_status")
