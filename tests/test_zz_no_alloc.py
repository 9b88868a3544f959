"""moe_route_noalloc: routing for callers that cannot allocate device memory
(a plugin handed only its input and output buffers, or code under an allocator
that owns the whole device pool).  Its scratch is a static array inside the
library instead of a caller workspace; its results must match moe_route's.

Collected last on purpose, so a failure here does not hide the other tests."""
import ctypes

import numpy as np
import pytest

from workloads import CONFIGS, MoEConfig, make_inputs


def _valid(layer_tensors, T, E):
    """Copy the parts of a routing that are defined (the pair and row arrays
    have unused tails)."""
    r = {k: v.cpu() for k, v in layer_tensors.items() if v is not None}
    P = int(r["tok_ptr"][T])
    R = int(r["offsets"][E])
    for k in ("pair_expert", "pair_gate", "pair_row"):
        r[k] = r[k][:P]
    for k in ("row_tok", "row_gate"):
        r[k] = r[k][:R]
    r["tile_expert"] = r["tile_expert"][:R // 128]
    return r


def test_rejects_shapes_beyond_the_static_scratch():
    from fine_grained_mixture_top_b200 import build
    build.build()
    from fine_grained_mixture_top_b200 import moe
    dims = moe.dims_of(4096, 8192, 1024, 64, 8)   # Wr split alone needs 48 MiB
    rt = moe.MoeRouting()
    rc = moe.lib().moe_route_noalloc(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, None,
                                     ctypes.byref(rt), None)
    assert rc == moe.MOE_ERR_SCRATCH_LIMIT
    assert "static" in moe.status_str(rc)


@pytest.mark.gpu
def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    import torch
    from fine_grained_mixture_top_b200 import moe
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [CONFIGS["tiny"],
             MoEConfig("noalloc2", T=3000, d=256, E=40, n=64, K=3, w_std=0.05, bias="normal", seed=41)]
    for i, cfg in enumerate(cases):        # two calls in a row, different shapes
        inp = make_inputs(cfg, "cuda", need_grad_inputs=False)
        ref = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
        # moe_route runs the same kernels first, so none of them is loaded
        # (lazily, by the CUDA driver) during the measured call below
        ref.route(inp["X"], inp["Wr"], inp["bias"])
        rt = moe.Routing.allocate(ref.dims, ref.sizes, "cuda")
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        moe.moe_route_noalloc(ref.dims, ref.opts, inp["X"], inp["Wr"], inp["bias"], rt)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        assert moe.moe_get_status() == (0, 0)
        if i > 0:
            # the first call resolved the static array's address (and may have
            # loaded the module that holds it); later calls take no device memory
            assert free1 == free0, (free0, free1)
        a = _valid(ref.routing.tensors, cfg.T, cfg.E)
        b = _valid(rt.tensors, cfg.T, cfg.E)
        assert a.keys() == b.keys()
        for k in a:
            if a[k].dtype == torch.int32:
                assert torch.equal(a[k], b[k]), k
            else:  # the floating-point tolerances of the parity tests
                tol = 1e-5 if k == "probs" else 1e-5 * float(a[k].abs().max()) + 1e-7
                assert float((a[k] - b[k]).abs().max()) <= tol, k
        np.testing.assert_array_equal(b["counts"].numpy().sum(), cfg.T * cfg.K)
