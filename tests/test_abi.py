"""The C-ABI library loads on a host without a GPU, exports every entry point
include/moe.h declares, and its host-only logic (shape checks, workspace
sizing, status strings) behaves as documented.  No compute call is made."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def moe():
    from fine_grained_mixture_top_b200 import build
    build.build()
    from fine_grained_mixture_top_b200 import moe as m
    return m


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:moe_status|const char\*)\s+(moe_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("moe_route", "moe_token_round", "moe_forward", "moe_backward", "moe_query_sizes",
              "moe_get_status", "moe_status_str"):
        assert s in syms


def test_library_exports_every_declared_symbol(moe):
    lib = moe.lib()
    for s in declared_symbols():
        assert hasattr(lib, s), s
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)$", out, re.M))
    assert set(declared_symbols()) <= exported


def test_query_sizes_matches_documented_capacities(moe):
    T, d, E, n, K = 16384, 1536, 128, 256, 8
    s = moe.query_sizes(moe.dims_of(T, d, E, n, K), moe.opts_of(0, 1, 0))
    assert s.P_max == T * K
    assert s.R_max % 128 == 0 and s.R_max >= T * K + 127 * E
    assert s.h_elems == s.R_max * 2 * n
    # forward workspace holds A [R,n] and Y [R,d] in bf16
    assert s.fwd_ws >= s.R_max * (n + d) * 2
    # token rounding enlarges the pair capacity by at most one tile per expert
    s2 = moe.query_sizes(moe.dims_of(T, d, E, n, K), moe.opts_of(2, 1, 7))
    assert s2.P_max == min(T * E, T * K + 127 * E)


@pytest.mark.parametrize("shape,code", [
    ((512, 100, 16, 64, 2), 2),    # d not a multiple of 128
    ((512, 128, 16, 48, 2), 2),    # n not a multiple of 64
    ((512, 128, 4, 64, 5), 2),     # K > E
    ((512, 128, 2048, 64, 2), 2),  # E > 1024
    ((512, 128, 64, 64, 33), 2),   # K > 32
    ((0, 128, 16, 64, 2), 2),      # no tokens
])
def test_query_sizes_rejects_unsupported_shapes(moe, shape, code):
    s = moe.MoeSizes()
    rc = moe.lib().moe_query_sizes(ctypes.byref(moe.dims_of(*shape)), ctypes.byref(moe.opts_of()), ctypes.byref(s))
    assert rc == code


def test_invalid_options_and_null_arguments(moe):
    L = moe.lib()
    s = moe.MoeSizes()
    dims = moe.dims_of(512, 128, 16, 64, 2)
    assert L.moe_query_sizes(ctypes.byref(dims), ctypes.byref(moe.opts_of(3, 1, 0)), ctypes.byref(s)) == 1
    assert L.moe_query_sizes(ctypes.byref(dims), ctypes.byref(moe.opts_of(0, 2, 0)), ctypes.byref(s)) == 1
    assert L.moe_query_sizes(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None) == 1
    # argument errors are caught on the host before any GPU call
    rt = moe.MoeRouting()
    assert L.moe_route(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, None, ctypes.byref(rt),
                       None, 0, None) == 1
    assert L.moe_forward(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, None, ctypes.byref(rt),
                         None, None, None, 0, None) == 1
    assert L.moe_set_spin_limit(10) == 1
    assert L.moe_set_sm_budget(-1) == 1
    assert L.moe_set_sm_budget(0) == 0
    assert L.moe_backward_ev(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, None, None, None,
                             ctypes.byref(rt), None, None, None, None, None, None, 0, None, None) == 1
    assert L.moe_mx_quantize_rows(None, 4, 32, None, None, None) == 1
    assert L.moe_mx_quantize_rows(None, 4, 48, None, None, None) == 2     # K not a multiple of 32
    assert L.moe_mx_quantize_cols(None, 1, 64, 8, None, None, None) == 1
    # MXFP8 forward: unsupported n (% 128) before anything else; then arguments
    assert L.moe_forward_mxfp8(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, None, ctypes.byref(rt),
                               None, None, None, 0, None) == 2
    dims128 = moe.dims_of(512, 128, 16, 128, 2)
    assert L.moe_forward_mxfp8(ctypes.byref(dims128), ctypes.byref(moe.opts_of()), None, None, None,
                               ctypes.byref(rt), None, None, None, 0, None) == 1
    assert moe.query_sizes(dims128, moe.opts_of()).fwd_mx_ws > 0
    assert moe.query_sizes(dims128, moe.opts_of()).mx_weights_bytes >= 3 * 16 * 128 * 128
    assert L.moe_mx_quantize_weights(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, None, 0, None) == 2
    assert L.moe_mx_quantize_weights(ctypes.byref(dims128), ctypes.byref(moe.opts_of()), None, None, None, 0,
                                     None) == 1
    assert L.moe_forward_mxfp8_q(ctypes.byref(dims128), ctypes.byref(moe.opts_of()), None, None, ctypes.byref(rt),
                                 None, None, None, 0, None) == 1
    assert moe.query_sizes(dims, moe.opts_of()).fwd_mx_ws == 0      # n = 64: no MXFP8 forward
    # expert-parallel and given-routing entry points
    assert L.moe_route_given(ctypes.byref(dims), ctypes.byref(moe.opts_of()), ctypes.byref(rt), None, 0, None) == 1
    assert L.moe_ep_pack(ctypes.byref(dims), ctypes.byref(moe.opts_of()), ctypes.byref(rt), None, None, None, None,
                         None, 0, None) == 1
    assert L.moe_ep_combine(ctypes.byref(dims), ctypes.byref(moe.opts_of()), ctypes.byref(rt), None, None, None,
                            None) == 1
    assert L.moe_router_backward(ctypes.byref(dims), ctypes.byref(moe.opts_of()), None, None, ctypes.byref(rt),
                                 None, None, None, None, None, 0, None) == 1
    assert L.moe_route_given(ctypes.byref(moe.dims_of(512, 100, 16, 64, 2)), ctypes.byref(moe.opts_of()),
                             ctypes.byref(rt), None, 0, None) == 2
    assert moe.last_error() == ""  # no CUDA error on this thread


def test_status_strings(moe):
    assert moe.status_str(0) == "ok"
    assert "timed out" in moe.status_str(5)
    assert moe.status_str(99) == "unknown status"


def _noalloc_bytes(T, d, E, K):
    """Scratch of moe_route_noalloc by the formula its header documents."""
    up = lambda x: -(-x // 256) * 256   # noqa: E731
    return (up(2 * d * 3 * (-(-E // 64) * 64)) + up(16) + up(4 * (-(-T // 256)) * E) + up(4 * T * K))


def test_route_noalloc_scratch_limit_follows_the_documented_formula():
    """Shapes the formula puts within 16 MiB get past the scratch check (and
    fail the null-pointer check); shapes just beyond it are refused."""
    import ctypes
    from fine_grained_mixture_top_b200 import moe
    limit = 16 << 20
    d, E, K = 1024, 64, 8
    # largest T (multiple of 8) that fits, by the formula
    T = 8
    while _noalloc_bytes(T + 8, d, E, K) <= limit:
        T += 8
    for t, fits in ((T, True), (T + 8, False), (T + 4096, False), (1000, True)):
        assert (_noalloc_bytes(t, d, E, K) <= limit) == fits
        rt = moe.MoeRouting()
        rc = moe.lib().moe_route_noalloc(ctypes.byref(moe.dims_of(t, d, E, 64, K)), ctypes.byref(moe.opts_of()),
                                         None, None, None, ctypes.byref(rt), None)
        assert rc == (moe.MOE_ERR_INVALID_ARG if fits else moe.MOE_ERR_SCRATCH_LIMIT), (t, rc)


def test_saved_activation_is_constant_in_granularity():
    """The only per-(token, expert) tensor kept from forward to backward is H
    [R, 2n] (moe_sizes.h_elems); neither Y nor A is kept.  At a fixed activated
    width K*n, making experts finer (E up, n down, K up) leaves it unchanged
    up to the 128-row padding of each expert's segment, while a layer that
    cached Y [T*K, d] would grow with K (page "DeepSeek做大→Mega MoE，Tri Dao团队
    加快→SonicMoE", section "第一，激活内存与专家粒度解耦"; the activation
    memory of the paper summary's results paragraph)."""
    from fine_grained_mixture_top_b200 import moe
    T, d = 16384, 1536
    family = [(64, 512, 4), (128, 256, 8), (256, 128, 16), (512, 64, 32)]   # K * n = 2048
    saved, y_cache = [], []
    for E, n, K in family:
        s = moe.query_sizes(moe.dims_of(T, d, E, n, K), moe.opts_of())
        assert s.h_elems == s.R_max * 2 * n
        # padding: at most 127 rows per expert, i.e. at most 127 E 2n = 254 E n elements
        assert 2 * T * K * n <= s.h_elems <= 2 * T * K * n + 254 * E * n + 2 * 128 * n
        saved.append(s.h_elems)
        y_cache.append(T * K * d)
    # 2 T K n = 2 T * 2048 on the whole family; padding adds at most 254 E n
    # (E n = 32768 throughout) plus the final round-up to 128 rows, under 13 %
    base = 2 * T * 2048
    for (E, n, K), h in zip(family, saved):
        assert base <= h <= base + 254 * E * n + 256 * n
    assert max(saved) / min(saved) < 1.13
    assert y_cache[-1] == 8 * y_cache[0]


def test_plan_log_prints_each_shape_once():
    """MOE_LOG=1 prints the tile plan of a new shape once on stderr (host
    only: moe_query_sizes plans without a GPU)."""
    code = (
        "import ctypes\n"
        "from fine_grained_mixture_top_b200 import moe\n"
        "s = moe.MoeSizes()\n"
        "for T in (4096, 4096, 8192):\n"
        "    assert moe.lib().moe_query_sizes(ctypes.byref(moe.dims_of(T, 1536, 128, 256, 8)),\n"
        "                                     ctypes.byref(moe.opts_of()), ctypes.byref(s)) == 0\n"
    )
    env = dict(os.environ, MOE_LOG="1")
    r = subprocess.run([os.sys.executable, "-c", code], capture_output=True, text=True, env=env,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), timeout=120)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stderr.splitlines() if ln.startswith("moe plan")]
    assert len(lines) == 2, r.stderr
    assert "T=4096 d=1536 E=128 n=256 K=8" in lines[0] and "router tile 384 columns" in lines[0]


def test_plan_choices_for_the_benchmark_layers():
    """The tile plan the measurements chose, per benchmark layer (host only:
    moe_query_sizes plans without a GPU; MOE_LOG=1 prints the plan): epilogue
    warps of dH / dX~ / the weight gradients, the 256-row down-proj tiles,
    the router tile width and the dWr split-K."""
    import re
    layers = {  # (T, d, E, n, K): (dH, dX~, dW warps, wide down, router columns, dWr splits)
        (8192, 7168, 256, 2048, 8): (4, 4, 4, 1, 384, 3),
        (16384, 1536, 128, 256, 8): (4, 4, 4, 0, 384, 6),
        (32768, 2048, 128, 768, 8): (4, 4, 4, 1, 384, None),
        (32768, 2048, 64, 1024, 8): (4, 4, 4, 1, 192, None),
        (16384, 1536, 256, 128, 8): (4, 8, 4, 0, 384, None),
        (16384, 1536, 512, 64, 8): (4, 8, 4, 0, 384, None),
        (512, 128, 16, 64, 2): (8, 8, 4, 0, 192, None),
    }
    code = (
        "import ctypes\n"
        "from fine_grained_mixture_top_b200 import moe\n"
        "s = moe.MoeSizes()\n"
        f"for T, d, E, n, K in {list(layers)!r}:\n"
        "    assert moe.lib().moe_query_sizes(ctypes.byref(moe.dims_of(T, d, E, n, K)),\n"
        "                                     ctypes.byref(moe.opts_of()), ctypes.byref(s)) == 0\n"
    )
    env = {k: v for k, v in os.environ.items() if not k.startswith("MOE_")}
    env["MOE_LOG"] = "1"
    r = subprocess.run([os.sys.executable, "-c", code], capture_output=True, text=True, env=env,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), timeout=120)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stderr.splitlines() if ln.startswith("moe plan")]
    assert len(lines) == len(layers), r.stderr
    for ln, ((T, d, E, n, K), want) in zip(lines, layers.items()):
        assert f"T={T} d={d} E={E} n={n} K={K}" in ln, ln
        warps = tuple(int(x) for x in re.search(r"epilogue warps dH (\d+) dX~ (\d+) dW (\d+)", ln).groups())
        wide = int(re.search(r"256-row tiles on one CTA down (\d+)", ln).group(1))
        rtr = int(re.search(r"router tile (\d+) columns", ln).group(1))
        splits = int(re.search(r"dWr split-K (\d+) x", ln).group(1))
        got = warps + (wide, rtr, splits if want[5] is not None else None)
        assert got == want, (ln, got, want)
