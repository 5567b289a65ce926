"""The C-ABI library on the host: exports, plan validation, argument checks.

Nothing here launches a kernel, so these run without a GPU.
"""
import ctypes
import os
import re

import pytest

from oracle import lighthouse as oracle
from long_context_hierarchical_b200 import lh
from long_context_hierarchical_b200.synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "lh.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lh_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_function_is_exported():
    names = declared_functions()
    assert len(names) >= 18
    lib = ctypes.CDLL(lh.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(lh.EXPORTS)


def test_plan_struct_matches_binding():
    assert lh.LIB.lh_plan_bytes() == ctypes.sizeof(lh.LhPlan)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_plan_sizes_match_oracle(name):
    w = WORKLOADS[name]
    p = lh.plan(w.B, w.H, w.N, w.d, w.p, w.L, w.k, w.dtype, select=w.select)
    sz = oracle.sizes(w.N, w.p, w.L, w.k)
    assert (p.S, p.M, p.Ntot, p.Ksel) == (sz.S, sz.M, sz.Ntot, sz.Ksel)
    assert list(p.raw.flat_off)[: w.L + 1] == sz.flat_off
    assert p.Npyr == sz.Ntot - w.N
    assert p.raw.ctx_bytes > 0 and p.raw.ws_bytes > 0
    for off in ("ctx_sel_idx", "ctx_slot_of", "ctx_Qg", "ctx_Kg", "ctx_Vg", "ctx_Og", "ctx_lse",
                "ws_pyrQ", "ws_scores", "ws_topk", "ws_dOg", "ws_D", "ws_attn"):
        assert getattr(p.raw, off) % 256 == 0


@pytest.mark.parametrize("args,status", [
    ((1, 2, 1000, 64, 4, 3, 1, "bf16"), lh.LH_ERR_INVALID_ARG),   # N % p^(L-1)
    ((1, 2, 1024, 64, 4, 3, 200, "bf16"), lh.LH_ERR_INVALID_ARG),  # budget > M
    ((1, 2, 1024, 64, 1, 3, 1, "bf16"), lh.LH_ERR_INVALID_ARG),    # p < 2
    ((1, 2, 1024, 64, 4, 0, 1, "bf16"), lh.LH_ERR_INVALID_ARG),    # L < 1
    ((0, 2, 1024, 64, 4, 3, 1, "bf16"), lh.LH_ERR_INVALID_ARG),    # B < 1
    ((1, 2, 1024, 64, 4, 3, -1, "bf16"), lh.LH_ERR_INVALID_ARG),   # k < 0
    ((1, 2, 1024, 96, 4, 3, 1, "bf16"), lh.LH_ERR_UNSUPPORTED),    # d = 96
    ((1, 2, 1024, 128, 4, 3, 1, "bf16"), None),                    # d = 128: built
    ((1, 2, 1152, 64, 3, 3, 1, "bf16"), lh.LH_ERR_UNSUPPORTED),    # p = 3
    ((1, 2, 4096, 64, 2, 6, 1, "bf16"), lh.LH_ERR_UNSUPPORTED),    # L = 6
    ((1, 2, 4096, 64, 4, 5, 1, "bf16"), None),                     # p^(L-1) = 256: built
    ((1, 65536, 64, 64, 4, 2, 1, "bf16"), lh.LH_ERR_UNSUPPORTED),  # B*H above the grid's y limit
    ((3, 21845, 64, 64, 4, 2, 1, "bf16"), None),                   # B*H = 65535: built
    ((1, 2048, 2**20, 64, 4, 1, 0, "bf16"), lh.LH_ERR_UNSUPPORTED),  # B*H*S = 2^31: TMA rows
    ((1, 2047, 2**20, 64, 4, 1, 0, "bf16"), None),                   # B*H*S < 2^31: built
    ((1, 2048, 2**20, 64, 4, 1, 0, "f32"), None),                    # fp32 has no TMA limit
])
def test_plan_validation(args, status):
    if status is None:
        lh.plan(*args)
        return
    with pytest.raises(lh.LighthouseError) as e:
        lh.plan(*args)
    assert e.value.status == status


def test_plan_regional_selection_option():
    """The regional rule keeps the same S and adds a candidate mask and the
    regions' leftover lists to the top-K scratch; an unknown rule is refused."""
    joint = lh.plan(1, 2, 8192, 64, 4, 4, 256, "bf16")
    reg = lh.plan(1, 2, 8192, 64, 4, 4, 256, "bf16", select="regional")
    assert reg.S == joint.S
    assert reg.raw.topk_ws_bytes >= joint.raw.topk_ws_bytes + 2 * reg.M
    cfg = lh.LhConfig(1, 2, 1024, 64, 4, 3, 8, lh.LH_BF16, 3)
    assert lh.LIB.lh_plan_init(ctypes.byref(cfg), ctypes.byref(lh.LhPlan())) == lh.LH_ERR_INVALID_ARG


def test_plan_descent_selection_option():
    """The descent rule keeps the same S, adds its scratch to the top-K
    workspace, and needs k <= N / p^(L-1)."""
    joint = lh.plan(1, 2, 1024, 64, 4, 3, 64, "bf16")
    desc = lh.plan(1, 2, 1024, 64, 4, 3, 64, "bf16", select="descent")  # n[2] = 64 = k
    assert desc.S == joint.S and desc.raw.c.select == 1
    assert desc.raw.topk_ws_bytes > joint.raw.topk_ws_bytes
    with pytest.raises(lh.LighthouseError) as e:
        lh.plan(1, 2, 1024, 64, 4, 3, 65, "bf16", select="descent")
    assert e.value.status == lh.LH_ERR_INVALID_ARG
    cfg = lh.LhConfig(1, 2, 1024, 64, 4, 3, 1, lh.LH_BF16, 7)
    assert lh.LIB.lh_plan_init(ctypes.byref(cfg), ctypes.byref(lh.LhPlan())) == lh.LH_ERR_INVALID_ARG
    assert b"select" in lh.LIB.lh_last_error()


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "lh.h"
int main(void) {
  lh_config c;
  lh_plan p;
  memset(&c, 0, sizeof c);
  c.B = 1; c.H = 16; c.N = 98304; c.d = 64; c.p = 4; c.L = 3; c.k = 1536;
  c.dtype = LH_BF16; c.select = LH_SELECT_JOINT;
  if (lh_plan_bytes() != (int64_t)sizeof(lh_plan)) return 2;
  if (lh_plan_init(&c, &p) != LH_OK) return 3;
  c.k = 1 << 20;
  if (lh_plan_init(&c, &p) != LH_ERR_INVALID_ARG) return 4;
  printf("%lld %lld %s\n", (long long)p.S, (long long)p.M, lh_status_string(LH_ERR_TIMEOUT));
  return 0;
}
"""


def test_header_compiles_as_c_and_links(tmp_path):
    """A plain C11 program includes lh.h and calls the host-only entry points
    of liblh.so (no GPU needed): the boundary is usable without PyTorch."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lh.LIB_PATH)
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        str(src), "-o", str(exe), "-L", libdir, "-llh", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    S, M, name = r.stdout.strip().split(maxsplit=2)
    assert (int(S), int(M)) == (18432, 122880)
    assert name == lh.LIB.lh_status_string(lh.LH_ERR_TIMEOUT).decode()


def test_plan_rejects_unknown_dtype():
    cfg = lh.LhConfig(1, 2, 1024, 64, 4, 3, 1, 7)
    out = lh.LhPlan()
    assert lh.LIB.lh_plan_init(ctypes.byref(cfg), ctypes.byref(out)) == lh.LH_ERR_UNSUPPORTED
    assert lh.LIB.lh_plan_init(None, ctypes.byref(out)) == lh.LH_ERR_INVALID_ARG


def test_entry_points_reject_bad_pointers_before_launching():
    p = lh.plan(1, 2, 1024, 64, 4, 3, 8, "bf16")
    ref = p.byref()
    good = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced here
    odd = ctypes.c_void_p((1 << 20) + 8)  # not 16-byte aligned
    L = lh.LIB
    cb, wb = p.raw.ctx_bytes, p.raw.ws_bytes
    assert L.lh_forward(ref, None, good, good, good, good, cb, good, wb, None) == lh.LH_ERR_INVALID_ARG
    assert L.lh_forward(ref, good, good, good, good, good, cb, odd, wb, None) == lh.LH_ERR_INVALID_ARG
    assert b"aligned" in L.lh_last_error()
    assert L.lh_backward(ref, good, None, cb, good, good, good, good, wb, None) == lh.LH_ERR_INVALID_ARG
    assert L.lh_topk(ref, good, good, good, good, 16, None) == lh.LH_ERR_WORKSPACE
    assert L.lh_attn_fwd(2, 100, 96, lh.LH_BF16, good, good, good, good, good, None) == lh.LH_ERR_UNSUPPORTED
    assert L.lh_attn_fwd(0, 100, 64, lh.LH_BF16, good, good, good, good, good, None) == lh.LH_ERR_INVALID_ARG
    assert L.lh_attn_bwd_ws_bytes(2, 100, 64, lh.LH_BF16) >= 2 * 100 * 4
    assert L.lh_attn_bwd(2, 100, 64, lh.LH_BF16, good, good, good, good, good, good, None, good,
                         good, good, good, 0, None) == lh.LH_ERR_WORKSPACE
    # a plan that was not produced by lh_plan_init is refused
    bad = lh.LhPlan.from_buffer_copy(p.raw)
    bad.S += 1
    assert L.lh_scatter(ctypes.byref(bad), good, good, good, None) == lh.LH_ERR_INVALID_ARG


def test_whole_layer_calls_check_buffer_sizes_before_launching():
    """lh_forward / lh_backward refuse a ctx or ws smaller than the plan's
    (LH_ERR_WORKSPACE, nothing enqueued); the pointers are never touched."""
    p = lh.plan(1, 2, 1024, 64, 4, 3, 8, "bf16")
    ref, L = p.byref(), lh.LIB
    good = ctypes.c_void_p(1 << 20)
    cb, wb = p.raw.ctx_bytes, p.raw.ws_bytes
    assert L.lh_forward(ref, good, good, good, good, good, cb - 1, good, wb, None) == lh.LH_ERR_WORKSPACE
    assert b"ctx_bytes" in L.lh_last_error()
    assert L.lh_forward(ref, good, good, good, good, good, cb, good, wb - 256, None) == lh.LH_ERR_WORKSPACE
    assert b"ws_bytes" in L.lh_last_error()
    assert L.lh_backward(ref, good, good, 0, good, good, good, good, wb, None) == lh.LH_ERR_WORKSPACE
    assert L.lh_backward(ref, good, good, cb, good, good, good, good, 16, None) == lh.LH_ERR_WORKSPACE


def test_status_strings():
    for s in range(6):
        assert lh.LIB.lh_status_string(s)


def test_binding_checks_tensor_arguments_before_calling_the_library():
    """The binding refuses a tensor of the wrong dtype, layout, size or device
    before any pointer reaches the library (a kernel would read or write past
    it)."""
    import torch
    pl = lh.plan(1, 2, 256, 64, 4, 3, 4, "bf16")
    tok = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    cases = [
        (lambda: lh.forward(pl, tok.float(), tok, tok), "dtype"),
        (lambda: lh.forward(pl, tok.transpose(2, 3), tok, tok), "contiguous"),
        (lambda: lh.forward(pl, tok[:, :1], tok, tok), "elements"),
        (lambda: lh.forward(pl, tok, tok, tok), "CUDA"),
        (lambda: lh.topk(pl, torch.zeros(1, 2, pl.M, dtype=torch.float64)), "dtype"),
        (lambda: lh.scatter(pl, torch.zeros(1, 2, pl.S, 64),
                            torch.zeros(1, 2, pl.Ntot, dtype=torch.int32)), "dtype"),
        (lambda: lh.gather_bwd(pl, *(torch.zeros(1, 2, pl.S - 1, 64, dtype=torch.bfloat16),) * 3,
                               torch.zeros(1, 2, pl.Ntot, dtype=torch.int32)), "elements"),
        (lambda: lh.attn_fwd(*(torch.zeros(2, 128, 64, dtype=torch.float16),) * 3), "dtype"),
        (lambda: lh.attn_fwd(torch.zeros(2, 128, 64).transpose(1, 2), None, None), "contiguous"),
        (lambda: lh.attn_bwd(torch.zeros(64), None, None, None, None, None), "[..., S, d]"),
        (lambda: lh.attn_fwd(*(torch.zeros(2, 128, 64),) * 3), "CUDA"),
        (lambda: lh.backward(pl, [0.0], None), "torch.Tensor"),
    ]
    for call, what in cases:
        with pytest.raises((ValueError, TypeError)) as e:
            call()
        assert what in str(e.value), (what, str(e.value))
