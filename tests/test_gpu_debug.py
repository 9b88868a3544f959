"""The debug build (libmoe_debug.so, MOE_DEBUG=1): device-side routing checks
that report through the status word instead of faulting.  Runs in a child
process, since one process loads one build of the library.

- On valid inputs the debug build reports no violation and its outputs are
  bit-for-bit those of the release build (the checks change no arithmetic).
- A routing whose row map is made inconsistent on the host side (one row's
  token id set past T) is caught by the check before any kernel uses it: the
  entry point returns MOE_ERR_DEVICE_CHECK and the status word says which
  check failed.  The corrupted id would be clamped by the debug gather too, so
  no copy can leave its tensor even if the check were skipped."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
from fine_grained_mixture_top_b200 import moe
from workloads import CONFIGS, MoEConfig, make_inputs
assert moe.LIB_PATH.endswith(LIBNAME), moe.LIB_PATH
out = {}
cases = [CONFIGS["tiny"], MoEConfig("dbg", T=1000, d=256, E=24, n=128, K=4, bias="normal", seed=7),
         MoEConfig("dbg_tr", T=700, d=128, E=12, n=64, K=3, bias="normal", seed=8, round_mode=2)]
for cfg in cases:
    inp = make_inputs(cfg, "cuda")
    L = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, round_mode=cfg.round_mode, seed=cfg.seed)
    L.step(inp["X"], inp["Wr"], inp["bias"], inp["W1"], inp["W2"], inp["dO"])
    torch.cuda.synchronize()
    assert moe.moe_get_status() == (0, 0), moe.moe_get_status()
    for k in ("O", "dX", "dW1", "dW2", "dWr"):
        out[cfg.name + "." + k] = getattr(L, k).cpu()
if CORRUPT:
    cfg = cases[1]
    inp = make_inputs(cfg, "cuda")
    L = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, seed=cfg.seed)
    L.route(inp["X"], inp["Wr"], inp["bias"])
    torch.cuda.synchronize()
    r0 = int(L.routing["pair_row"][0])       # a real row (token 0's first pair)
    L.routing["row_tok"][r0] = cfg.T + 5
    torch.cuda.synchronize()
    try:
        L.forward(inp["X"], inp["W1"], inp["W2"])
        raise SystemExit("forward accepted a corrupt routing")
    except moe.MoEError as e:
        assert e.code == moe.MOE_ERR_DEVICE_CHECK, e
    code, where = moe.moe_get_status()
    assert code == moe.MOE_ERR_DEVICE_CHECK and 0x101 <= where <= 0x10B, (code, hex(where))
    out["corrupt_where"] = where
torch.save(out, OUT)
'''


def _run(tmp_path, debug, corrupt):
    out = tmp_path / ("debug.pt" if debug else "release.pt")
    env = dict(os.environ)
    env["MOE_DEBUG"] = "1" if debug else "0"
    code = (f"ROOT = {ROOT!r}; OUT = {str(out)!r}; LIBNAME = {'libmoe_debug.so' if debug else 'libmoe.so'!r}; "
            f"CORRUPT = {corrupt}\n" + CHILD)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    import torch
    return torch.load(out)


@pytest.mark.gpu
def test_debug_build_checks_routing_and_matches_release(tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fine_grained_mixture_top_b200 import build
    build.build(debug=True)
    dbg = _run(tmp_path, True, True)
    rel = _run(tmp_path, False, False)
    assert 0x101 <= dbg.pop("corrupt_where") <= 0x10B
    assert dbg.keys() == rel.keys()
    for k in rel:
        assert torch.equal(dbg[k], rel[k]), k
