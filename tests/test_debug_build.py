"""The FA_DEBUG build: the same kernels with device-side argument checks on
every TMA copy, tensor-memory access and MMA.  On the CPU: it builds and exports
what include/fa.h declares.  On a GPU: every kernel family runs through it on
small ragged shapes without a failed check, and its outputs are those of the
release build."""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from test_abi import _declared  # noqa: E402


def test_debug_library_builds_and_exports():
    from exact_io_aware_85_b200 import build
    lib = ctypes.CDLL(build.build_library(debug=True))
    for n in _declared():
        assert hasattr(lib, n), n
    lib.fa_status_string.restype = ctypes.c_char_p
    assert lib.fa_status_string(6) == b"FA_ERR_CHECK"


_SCRIPT = r"""
import math, sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from exact_io_aware_85_b200 import fa, synth
assert fa._DEBUG == (sys.argv[2] == "debug")
out = {}
def t(x, dt="bf16"):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16 if dt == "bf16" else torch.float32).cuda()
for d, N, causal in ((64, 333, True), (128, 200, False), (256, 129, True)):
    x = synth.make_inputs(1, 2, N, d, "bf16", seed=d + N, with_grad=True)
    q, k, v, do = (t(x[n]) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q); lse = torch.empty((1, 2, N), device="cuda")
    fa.fa_fwd(q, k, v, o, lse, causal, 1 / math.sqrt(d))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(1, 2, N, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, causal, 1 / math.sqrt(d), ws)
    torch.cuda.synchronize()
    out[f"fwd{d}"] = (o.float().cpu().numpy(), lse.cpu().numpy())
    out[f"bwd{d}"] = (dq.float().cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy())
    assert fa.fa_check_status() == 0, ("status", d)
x = synth.make_inputs(1, 2, 200, 64, "f32", seed=5)
q, k, v = (t(x[n], "f32") for n in ("q", "k", "v"))
o = torch.empty_like(q); lse = torch.empty((1, 2, 200), device="cuda")
fa.fa_fwd_f32(q, k, v, o, lse, True, 0.125)
torch.cuda.synchronize(); out["f32"] = (o.cpu().numpy(), lse.cpu().numpy())
x = synth.make_sink_inputs(1, 2, 300, 128, 8.0, seed=6)
q, k, v = (t(x[n]) for n in ("q", "k", "v"))
o = torch.empty_like(q); lse = torch.empty((1, 2, 300), device="cuda")
st = torch.zeros(4, dtype=torch.int64, device="cuda")
fa.fa_fwd_fp8p(q, k, v, o, lse, False, 1 / math.sqrt(128), 256.0, 1, st, 4)
torch.cuda.synchronize(); out["fp8p"] = (o.float().cpu().numpy(), st.cpu().numpy())
nb = 3
q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device="cuda") for _ in range(3))
sq, sk = (torch.empty((1, 2, nb), device="cuda") for _ in range(2)); sv = torch.empty((1, 2), device="cuda")
signs = torch.from_numpy(synth.random_signs(128, seed=1)).cuda()
fa.fa_fp8_quantize(q, k, v, signs, q8, k8, v8, sq, sk, sv)
fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, True, 1 / math.sqrt(128), 256.0, 0)
torch.cuda.synchronize(); out["fp8"] = (o.float().cpu().numpy(),)
for dd, nn in ((64, 200), (256, 150)):  # 64-byte E4M3 rows; the 64-key-tile kernel
    x = synth.make_inputs(1, 2, nn, dd, "bf16", seed=dd + 3)
    q, k, v = (t(x[n]) for n in ("q", "k", "v"))
    o = torch.empty_like(q); lse = torch.empty((1, 2, nn), device="cuda")
    nb = (nn + 127) // 128
    q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device="cuda") for _ in range(3))
    sq, sk = (torch.empty((1, 2, nb), device="cuda") for _ in range(2)); sv = torch.empty((1, 2), device="cuda")
    fa.fa_fp8_quantize(q, k, v, None, q8, k8, v8, sq, sk, sv)
    fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, True, 1 / math.sqrt(dd), 256.0, 1)
    torch.cuda.synchronize(); out[f"fp8_{dd}"] = (o.float().cpu().numpy(),)
    if dd == 256:
        st = torch.zeros(4, dtype=torch.int64, device="cuda")
        fa.fa_fwd_fp8p(q, k, v, o, lse, True, 1 / math.sqrt(dd), 256.0, 1, st, 4)
        torch.cuda.synchronize(); out["fp8p_256"] = (o.float().cpu().numpy(), st.cpu().numpy())
xd = synth.make_inputs(2, 4, 1000, 128, "bf16", seed=7)
qd = t(xd["q"][:, :, 0]); kd, vd = t(xd["k"][:, :2]), t(xd["v"][:, :2])
od = torch.empty_like(qd); lsed = torch.empty((2, 4), device="cuda")
wsd = torch.empty(fa.fa_decode_workspace_bytes(2, 4, 2, 1000, 128), dtype=torch.uint8, device="cuda")
fa.fa_decode(qd, kd, vd, od, lsed, 1 / math.sqrt(128), wsd)
torch.cuda.synchronize(); out["decode"] = (od.float().cpu().numpy(), lsed.cpu().numpy())
assert fa.fa_check_status() == 0, "status"
np.savez(sys.argv[3], **{f"{k}_{i}": a for k, v in out.items() for i, a in enumerate(v)})
"""


@pytest.mark.gpu
def test_debug_build_checks_pass_and_matches_release(tmp_path):
    from exact_io_aware_85_b200 import build
    build.build_library(debug=True)
    res = {}
    for mode in ("release", "debug"):
        env = dict(os.environ, FA_DEBUG="1" if mode == "debug" else "0")
        path = str(tmp_path / f"{mode}.npz")
        r = subprocess.run([sys.executable, "-c", _SCRIPT, ROOT, mode, path], env=env, capture_output=True,
                           text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        res[mode] = dict(np.load(path))
    for key, a in res["release"].items():
        b = res["debug"][key]
        if key.startswith("bwd") and key.endswith("_0"):  # dQ: fp32 reductions in arrival order
            assert np.abs(a - b).max() <= 1e-2 * max(1.0, np.abs(a).max()), key
        else:
            assert np.array_equal(a, b), key
