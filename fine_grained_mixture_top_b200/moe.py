"""Python binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; torch supplies the
device memory and the stream.  There is no fallback: if the shared library is
missing the import of this module's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_DEBUG=1 in the environment loads the debug build instead (device-side
# routing checks reported through moe_get_status; same results otherwise)
LIB_PATH = os.path.join(_PKG, "libmoe_debug.so" if os.environ.get("MOE_DEBUG") == "1" else "libmoe.so")

c_void_p = ctypes.c_void_p
c_int32 = ctypes.c_int32
c_int64 = ctypes.c_int64

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, \
    MOE_ERR_DEVICE_CHECK, MOE_ERR_SCRATCH_LIMIT = range(8)


class MoeDims(ctypes.Structure):
    _fields_ = [("T", c_int64), ("d", c_int32), ("E", c_int32), ("n", c_int32), ("K", c_int32)]


class MoeOpts(ctypes.Structure):
    _fields_ = [("round_mode", c_int32), ("router_grad", c_int32), ("seed", ctypes.c_uint64)]


_ROUTING_PTRS = ["logits", "probs", "topk_idx", "topk_gate", "tok_ptr", "pair_expert", "pair_gate", "pair_row",
                 "counts", "offsets", "row_tok", "row_gate", "tile_expert"]


class MoeRouting(ctypes.Structure):
    _fields_ = [(name, c_void_p) for name in _ROUTING_PTRS] + [("P_max", c_int64), ("R_max", c_int64),
                                                                ("pair_dS", c_void_p)]


class MoeSizes(ctypes.Structure):
    _fields_ = [("P_max", c_int64), ("R_max", c_int64), ("route_ws", ctypes.c_size_t),
                ("fwd_ws", ctypes.c_size_t), ("bwd_ws", ctypes.c_size_t), ("h_elems", c_int64),
                ("fwd_mx_ws", ctypes.c_size_t), ("mx_weights_bytes", ctypes.c_size_t)]


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {status_str(code)} ({code})"
        if code == MOE_ERR_CUDA:
            msg += f": {last_error()}"
        super().__init__(msg)
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by fine_grained_mixture_top_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run python -m "
                               "fine_grained_mixture_top_b200.build" +
                               (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.moe_query_sizes.argtypes = [P(MoeDims), P(MoeOpts), P(MoeSizes)]
        L.moe_route.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, c_void_p, P(MoeRouting), c_void_p,
                                ctypes.c_size_t, c_void_p]
        L.moe_route_noalloc.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, c_void_p, P(MoeRouting),
                                         c_void_p]
        L.moe_route_noalloc.restype = c_int32
        L.moe_token_round.argtypes = [P(MoeDims), P(MoeOpts), P(MoeRouting), c_void_p, ctypes.c_size_t, c_void_p]
        L.moe_forward.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, c_void_p, P(MoeRouting), c_void_p,
                                  c_void_p, c_void_p, ctypes.c_size_t, c_void_p]
        L.moe_forward_mxfp8.argtypes = L.moe_forward.argtypes
        L.moe_mx_quantize_weights.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, c_void_p, ctypes.c_size_t,
                                              c_void_p]
        L.moe_forward_mxfp8_q.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, P(MoeRouting), c_void_p,
                                          c_void_p, c_void_p, ctypes.c_size_t, c_void_p]
        L.moe_backward.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   P(MoeRouting), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   ctypes.c_size_t, c_void_p]
        L.moe_backward_ev.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      P(MoeRouting), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      ctypes.c_size_t, P(c_void_p), c_void_p]
        L.moe_set_sm_budget.argtypes = [c_int32]
        L.moe_route_given.argtypes = [P(MoeDims), P(MoeOpts), P(MoeRouting), c_void_p, ctypes.c_size_t, c_void_p]
        L.moe_ep_pack.argtypes = [P(MoeDims), P(MoeOpts), P(MoeRouting), c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, ctypes.c_size_t, c_void_p]
        L.moe_ep_combine.argtypes = [P(MoeDims), P(MoeOpts), P(MoeRouting), c_void_p, c_void_p, c_void_p, c_void_p]
        L.moe_router_backward.argtypes = [P(MoeDims), P(MoeOpts), c_void_p, c_void_p, P(MoeRouting), c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_void_p, ctypes.c_size_t, c_void_p]
        L.moe_mx_quantize_rows.argtypes = [c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p]
        L.moe_mx_quantize_cols.argtypes = [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p]
        L.moe_get_status.argtypes = [c_void_p, P(c_int32)]
        L.moe_set_spin_limit.argtypes = [c_int64]
        L.moe_selftest_wait_timeout.argtypes = [c_void_p, c_void_p]
        L.moe_profile_enable.argtypes = [c_int32]
        L.moe_profile_enable.restype = c_int32
        L.moe_profile_select.argtypes = [ctypes.c_char_p]
        L.moe_profile_select.restype = c_int32
        L.moe_profile_count.argtypes = []
        L.moe_profile_count.restype = c_int32
        L.moe_profile_read.argtypes = [c_int32, P(ctypes.c_char_p), P(ctypes.c_float)]
        L.moe_profile_read.restype = c_int32
        L.moe_trace_gemm.argtypes = [c_int32, c_void_p, c_int64]
        L.moe_trace_gemm.restype = c_int32
        L.moe_status_str.argtypes = [c_int32]
        L.moe_status_str.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        for f in ("moe_query_sizes", "moe_route", "moe_token_round", "moe_forward", "moe_backward",
                  "moe_get_status", "moe_set_spin_limit", "moe_selftest_wait_timeout", "moe_backward_ev",
                  "moe_set_sm_budget", "moe_mx_quantize_rows", "moe_mx_quantize_cols", "moe_forward_mxfp8",
                  "moe_route_given", "moe_ep_pack", "moe_ep_combine", "moe_router_backward",
                  "moe_mx_quantize_weights", "moe_forward_mxfp8_q"):
            getattr(L, f).restype = c_int32
        _lib = L
    return _lib


def status_str(code: int) -> str:
    return lib().moe_status_str(int(code)).decode()


def last_error() -> str:
    """The CUDA runtime error behind this thread's most recent MOE_ERR_CUDA."""
    return lib().moe_last_error().decode()


def _check(code: int, what: str):
    if code != MOE_OK:
        raise MoEError(code, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def dims_of(T, d, E, n, K) -> MoeDims:
    return MoeDims(int(T), int(d), int(E), int(n), int(K))


def opts_of(round_mode=0, router_grad=1, seed=0) -> MoeOpts:
    return MoeOpts(int(round_mode), int(router_grad), int(seed))


def query_sizes(dims: MoeDims, opts: MoeOpts) -> MoeSizes:
    s = MoeSizes()
    _check(lib().moe_query_sizes(ctypes.byref(dims), ctypes.byref(opts), ctypes.byref(s)), "moe_query_sizes")
    return s


@dataclass
class Routing:
    """Device buffers of a moe_routing, allocated with torch."""
    tensors: dict
    struct: MoeRouting

    def __getitem__(self, k):
        return self.tensors[k]

    @classmethod
    def allocate(cls, dims: MoeDims, sizes: MoeSizes, device="cuda", with_logits: bool = True,
                 with_pair_ds: bool = False) -> "Routing":
        import torch
        T, E, K = dims.T, dims.E, dims.K
        P, R = sizes.P_max, sizes.R_max
        i32, f32 = torch.int32, torch.float32
        shapes = {"logits": ((T, E), f32), "probs": ((T, E), f32), "topk_idx": ((T, K), i32),
                  "topk_gate": ((T, K), f32), "tok_ptr": ((T + 1,), i32), "pair_expert": ((P,), i32),
                  "pair_gate": ((P,), f32), "pair_row": ((P,), i32), "counts": ((E,), i32),
                  "offsets": ((E + 1,), i32), "row_tok": ((R,), i32), "row_gate": ((R,), f32),
                  "tile_expert": ((R // 128,), i32)}
        t = {}
        for k, (shape, dt) in shapes.items():
            if k == "logits" and not with_logits:
                t[k] = None
                continue
            t[k] = torch.empty(shape, dtype=dt, device=device)
        t["pair_dS"] = torch.empty((P,), dtype=f32, device=device) if with_pair_ds else None
        st = MoeRouting(*[_ptr(t[k]) for k in _ROUTING_PTRS], P, R, _ptr(t["pair_dS"]))
        return cls(t, st)


def moe_route(dims, opts, X, Wr, bias, routing: Routing, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(dims), ctypes.byref(opts), _ptr(X), _ptr(Wr), _ptr(bias),
                           ctypes.byref(routing.struct), _ptr(ws), ws.numel() * ws.element_size(),
                           _stream(stream)), "moe_route")


def moe_route_given(dims, opts, routing: Routing, ws, stream=None):
    """Permutation of a caller-given selection (routing['topk_idx'],
    routing['topk_gate'] filled by the caller)."""
    _check(lib().moe_route_given(ctypes.byref(dims), ctypes.byref(opts), ctypes.byref(routing.struct), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "moe_route_given")


def moe_ep_pack(dims, opts, routing: Routing, src, send_rows, send_gate, pair_pos, ws, stream=None):
    _check(lib().moe_ep_pack(ctypes.byref(dims), ctypes.byref(opts), ctypes.byref(routing.struct), _ptr(src),
                             _ptr(send_rows), _ptr(send_gate), _ptr(pair_pos), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "moe_ep_pack")


def moe_ep_combine(dims, opts, routing: Routing, pair_pos, rows, out, stream=None):
    _check(lib().moe_ep_combine(ctypes.byref(dims), ctypes.byref(opts), ctypes.byref(routing.struct),
                                _ptr(pair_pos), _ptr(rows), _ptr(out), _stream(stream)), "moe_ep_combine")


def moe_router_backward(dims, opts, X, Wr, routing: Routing, dS, pair_pos, dX, dWr, ws, stream=None):
    _check(lib().moe_router_backward(ctypes.byref(dims), ctypes.byref(opts), _ptr(X), _ptr(Wr),
                                     ctypes.byref(routing.struct), _ptr(dS), _ptr(pair_pos), _ptr(dX), _ptr(dWr),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_router_backward")


def moe_route_noalloc(dims, opts, X, Wr, bias, routing: Routing, stream=None):
    """moe_route without a workspace, for callers that cannot allocate device
    memory; its scratch is a 16 MiB static array in the library (see moe.h)."""
    _check(lib().moe_route_noalloc(ctypes.byref(dims), ctypes.byref(opts), _ptr(X), _ptr(Wr), _ptr(bias),
                                   ctypes.byref(routing.struct), _stream(stream)), "moe_route_noalloc")


def moe_token_round(dims, opts, routing: Routing, ws, stream=None):
    _check(lib().moe_token_round(ctypes.byref(dims), ctypes.byref(opts), ctypes.byref(routing.struct), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "moe_token_round")


def moe_forward(dims, opts, X, W1, W2, routing: Routing, O, H, ws, stream=None):
    _check(lib().moe_forward(ctypes.byref(dims), ctypes.byref(opts), _ptr(X), _ptr(W1), _ptr(W2),
                             ctypes.byref(routing.struct), _ptr(O), _ptr(H), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "moe_forward")


def moe_forward_mxfp8(dims, opts, X, W1, W2, routing: Routing, O, H, ws, stream=None):
    _check(lib().moe_forward_mxfp8(ctypes.byref(dims), ctypes.byref(opts), _ptr(X), _ptr(W1), _ptr(W2),
                                   ctypes.byref(routing.struct), _ptr(O), _ptr(H), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "moe_forward_mxfp8")


def moe_mx_quantize_weights(dims, opts, W1, W2, wq, stream=None):
    _check(lib().moe_mx_quantize_weights(ctypes.byref(dims), ctypes.byref(opts), _ptr(W1), _ptr(W2), _ptr(wq),
                                         wq.numel() * wq.element_size(), _stream(stream)), "moe_mx_quantize_weights")


def moe_forward_mxfp8_q(dims, opts, X, wq, routing: Routing, O, H, ws, stream=None):
    _check(lib().moe_forward_mxfp8_q(ctypes.byref(dims), ctypes.byref(opts), _ptr(X), _ptr(wq),
                                     ctypes.byref(routing.struct), _ptr(O), _ptr(H), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "moe_forward_mxfp8_q")


def moe_backward(dims, opts, dO, X, Wr, W1, W2, routing: Routing, H, dX, dW1, dW2, dWr, ws, stream=None,
                 grad_events=None):
    """grad_events: None, or three torch.cuda.Event (or None) recorded once
    dW2, dW1 and dWr are final."""
    args = (ctypes.byref(dims), ctypes.byref(opts), _ptr(dO), _ptr(X), _ptr(Wr), _ptr(W1), _ptr(W2),
            ctypes.byref(routing.struct), _ptr(H), _ptr(dX), _ptr(dW1), _ptr(dW2), _ptr(dWr), _ptr(ws),
            ws.numel() * ws.element_size())
    if grad_events is None:
        _check(lib().moe_backward(*args, _stream(stream)), "moe_backward")
        return
    for e in grad_events:
        if e is not None and not e.cuda_event:  # torch creates its event on the first record
            e.record()
    evs = (c_void_p * 3)(*[None if e is None else e.cuda_event for e in grad_events])
    _check(lib().moe_backward_ev(*args, evs, _stream(stream)), "moe_backward_ev")


def mx_quantize_rows(x, stream=None):
    """x [rows, K] bf16 (device) -> (codes [rows, K] uint8, scales [rows, K/32]
    uint8): MXFP8 along each row."""
    import torch
    rows, K = x.shape
    codes = torch.empty(rows, K, dtype=torch.uint8, device=x.device)
    scales = torch.empty(rows, K // 32, dtype=torch.uint8, device=x.device)
    _check(lib().moe_mx_quantize_rows(_ptr(x), rows, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_mx_quantize_rows")
    return codes, scales


def mx_quantize_cols(w, stream=None):
    """w [E, K, N] bf16 (device) -> (codes [E, N, K] uint8, scales [E, N, K/32]
    uint8): MXFP8 along K for each column, transposed so that K is contiguous."""
    import torch
    E, K, N = w.shape
    codes = torch.empty(E, N, K, dtype=torch.uint8, device=w.device)
    scales = torch.empty(E, N, K // 32, dtype=torch.uint8, device=w.device)
    _check(lib().moe_mx_quantize_cols(_ptr(w), E, K, N, _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_mx_quantize_cols")
    return codes, scales


def moe_set_sm_budget(sms: int):
    """At most `sms` CTAs per persistent GEMM (0: one per SM)."""
    _check(lib().moe_set_sm_budget(int(sms)), "moe_set_sm_budget")


def moe_get_status(stream=None) -> tuple[int, int]:
    where = c_int32(0)
    code = lib().moe_get_status(_stream(stream), ctypes.byref(where))
    return int(code), int(where.value)


def moe_set_spin_limit(cycles: int):
    _check(lib().moe_set_spin_limit(int(cycles)), "moe_set_spin_limit")


def moe_selftest_wait_timeout(flag, stream=None):
    _check(lib().moe_selftest_wait_timeout(_ptr(flag), _stream(stream)), "moe_selftest_wait_timeout")


def moe_profile_enable(on: bool):
    _check(lib().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def moe_profile_select(name: str | None):
    """Record only launches of `name` (None: record every launch)."""
    _check(lib().moe_profile_select(None if name is None else name.encode()), "moe_profile_select")


def moe_profile_records() -> list[tuple[str, float]]:
    """(kernel name, ms) of every launch recorded since moe_profile_enable(True);
    the streams must have completed."""
    L = lib()
    out = []
    name = ctypes.c_char_p()
    ms = ctypes.c_float()
    for i in range(L.moe_profile_count()):
        _check(L.moe_profile_read(i, ctypes.byref(name), ctypes.byref(ms)), "moe_profile_read")
        out.append((name.value.decode(), float(ms.value)))
    return out


GEMM_KINDS = {"up_proj_gemm": 0, "down_proj_gemm": 1, "dh_gemm": 2, "dxt_gemm": 3, "dw1_gemm": 4, "dw2_gemm": 5,
              "router_logits_gemm": 6, "router_dwr_gemm": 7, "up_proj_gemm_mx": 8, "down_proj_gemm_mx": 9}


class GemmTrace:
    """Role timeline of one grouped-GEMM kind (moe_trace_gemm): start() before
    the launches to trace, stop() after them, then records() gives one numpy
    structured array per (CTA, role) with fields ns, clk, tile, event."""

    ROLES = ("producer", "mma", "epilogue", "gather")

    def __init__(self, kernel: str, records_per_role: int = 4096, device="cuda"):
        import torch
        self.kind = GEMM_KINDS[kernel]
        self.cap = int(records_per_role)
        sms = torch.cuda.get_device_properties(torch.device(device)).multi_processor_count
        self.ctas = sms
        self.buf = torch.zeros(self.ctas * 4 * self.cap * 16, dtype=torch.uint8, device=device)

    def start(self):
        self.buf.zero_()
        _check(lib().moe_trace_gemm(self.kind, _ptr(self.buf), self.cap), "moe_trace_gemm")

    def stop(self):
        _check(lib().moe_trace_gemm(-1, None, 0), "moe_trace_gemm")

    def records(self):
        import numpy as np
        raw = self.buf.cpu().numpy()
        dt = np.dtype([("ns", "<u8"), ("clk", "<u4"), ("info", "<u4")])
        rec = raw.view(dt).reshape(self.ctas, 4, self.cap)
        out = {}
        for c in range(self.ctas):
            for r in range(4):
                x = rec[c, r]
                x = x[x["ns"] != 0]
                out[(c, self.ROLES[r])] = {"ns": x["ns"].astype(np.int64), "clk": x["clk"].astype(np.int64),
                                           "tile": (x["info"] >> 8).astype(np.int64),
                                           "event": (x["info"] & 0xFF).astype(np.int64)}
        return out


class MoELayer:
    """All device buffers of one layer shape, allocated once with torch; each
    method is one library call."""

    def __init__(self, T, d, E, n, K, round_mode=0, router_grad=1, seed=0, device="cuda"):
        import torch
        self.dims = dims_of(T, d, E, n, K)
        self.opts = opts_of(round_mode, router_grad, seed)
        self.sizes = query_sizes(self.dims, self.opts)
        self.device = device
        self.routing = Routing.allocate(self.dims, self.sizes, device)
        u8, bf = torch.uint8, torch.bfloat16
        self.ws_route = torch.empty(self.sizes.route_ws, dtype=u8, device=device)
        self.ws_fwd = torch.empty(self.sizes.fwd_ws, dtype=u8, device=device)
        self.ws_bwd = torch.empty(self.sizes.bwd_ws, dtype=u8, device=device)
        self.ws_fwd_mx = None   # MXFP8 forward workspace, allocated on first use
        self.mxfp8 = False      # default precision of forward(): MXFP8 GEMM operands when True
        self.H = torch.empty(self.sizes.R_max, 2 * n, dtype=bf, device=device)
        self.O = torch.empty(T, d, dtype=bf, device=device)
        self.dX = torch.empty(T, d, dtype=bf, device=device)
        self.dW1 = torch.empty(E, d, 2 * n, dtype=bf, device=device)
        self.dW2 = torch.empty(E, n, d, dtype=bf, device=device)
        self.dWr = torch.empty(d, E, dtype=torch.float32, device=device)

    def route(self, X, Wr, bias=None, stream=None):
        moe_route(self.dims, self.opts, X, Wr, bias, self.routing, self.ws_route, stream)
        if self.opts.round_mode:
            moe_token_round(self.dims, self.opts, self.routing, self.ws_route, stream)

    def forward(self, X, W1, W2, stream=None, O=None, mxfp8=None):
        O = self.O if O is None else O
        if self.mxfp8 if mxfp8 is None else mxfp8:
            if self.ws_fwd_mx is None:
                import torch
                if self.sizes.fwd_mx_ws == 0:
                    raise MoEError(2, "moe_forward_mxfp8 (needs n % 128 == 0)")
                self.ws_fwd_mx = torch.empty(self.sizes.fwd_mx_ws, dtype=torch.uint8, device=self.device)
            moe_forward_mxfp8(self.dims, self.opts, X, W1, W2, self.routing, O, self.H, self.ws_fwd_mx, stream)
        else:
            moe_forward(self.dims, self.opts, X, W1, W2, self.routing, O, self.H, self.ws_fwd, stream)
        return O

    def quantize_weights_mxfp8(self, W1, W2, stream=None):
        """MXFP8 copy of W1, W2 for forward_mxfp8_q (weights that stay fixed)."""
        import torch
        if self.sizes.mx_weights_bytes == 0:
            raise MoEError(2, "moe_mx_quantize_weights (needs n % 128 == 0)")
        wq = torch.empty(self.sizes.mx_weights_bytes, dtype=torch.uint8, device=self.device)
        moe_mx_quantize_weights(self.dims, self.opts, W1, W2, wq, stream)
        return wq

    def forward_mxfp8_q(self, X, wq, stream=None, O=None):
        """The MXFP8 forward on weights quantized once by quantize_weights_mxfp8."""
        import torch
        O = self.O if O is None else O
        if self.ws_fwd_mx is None:
            self.ws_fwd_mx = torch.empty(self.sizes.fwd_mx_ws, dtype=torch.uint8, device=self.device)
        moe_forward_mxfp8_q(self.dims, self.opts, X, wq, self.routing, O, self.H, self.ws_fwd_mx, stream)
        return O

    def backward(self, dO, X, Wr, W1, W2, stream=None, grad_events=None, dX=None):
        """dX: output buffer [T, d] bf16 (default: self.dX)."""
        dX = self.dX if dX is None else dX
        moe_backward(self.dims, self.opts, dO, X, Wr, W1, W2, self.routing, self.H, dX, self.dW1, self.dW2,
                     self.dWr if self.opts.router_grad else None, self.ws_bwd, stream, grad_events)
        return dX, self.dW1, self.dW2, self.dWr

    def step(self, X, Wr, bias, W1, W2, dO, stream=None, grad_events=None):
        """One pass of the whole path: route (+ rounding), forward, backward."""
        self.route(X, Wr, bias, stream)
        self.forward(X, W1, W2, stream)
        return self.backward(dO, X, Wr, W1, W2, stream, grad_events)


class CudaStreamHooks:
    """Stream and event plumbing of OverlappedGradReduce on a CUDA device:
    three events the backward records (dW2, dW1, dWr written), and a
    communication stream that waits on each before its all-reduce."""

    def __init__(self):
        import torch
        self.comm = torch.cuda.Stream()
        self.events = [torch.cuda.Event() for _ in range(3)]

    def on_comm(self):
        import torch
        return torch.cuda.stream(self.comm)

    def wait(self, ev):
        self.comm.wait_event(ev)

    def join(self):
        import torch
        torch.cuda.current_stream().wait_stream(self.comm)


class OverlappedGradReduce:
    """Data-parallel steps whose weight-gradient sums over `group` overlap the
    backward.  The backward records an event as soon as dW2, then dW1, then dWr
    are written (moe_backward_ev computes dW2 and dW1 before dX~); each
    all-reduce waits on its event on a separate stream, so the reductions of
    dW2 and dW1 run while the dX~ GEMM and the dX aggregation do.  The current
    stream waits for the reductions at the end of the step, before the next
    step can overwrite the gradients.

    `hooks` supplies the streams and events (CudaStreamHooks by default); the
    CPU tests pass host stand-ins so that the ordering logic runs on gloo
    ranks."""

    def __init__(self, layer, group=None, hooks=None):
        self.layer = layer
        self.group = group
        self.hooks = hooks if hooks is not None else CudaStreamHooks()

    def step(self, X, Wr, bias, W1, W2, dO):
        import torch.distributed as dist
        L = self.layer
        h = self.hooks
        L.step(X, Wr, bias, W1, W2, dO, grad_events=h.events)
        grads = (L.dW2, L.dW1, L.dWr if L.opts.router_grad else None)
        with h.on_comm():
            for ev, g in zip(h.events, grads):
                if g is None:
                    continue
                h.wait(ev)
                dist.all_reduce(g, group=self.group)
        h.join()
        return L.dX, L.dW1, L.dW2, L.dWr


class HostFedRunner:
    """Whole steps (route, forward, backward) on batches held in pinned host
    memory.  Each step's inputs X and dO are copied to the device on a copy
    stream; its per-token outputs O and dX are copied back on a second copy
    stream, O as soon as the forward is done and dX after the backward, so the
    copies of consecutive steps overlap with the kernels.  Device input and
    output buffers alternate between two sets; events keep a buffer from being
    overwritten while a step or a copy still uses it.  Weight gradients stay
    on the device (layer.dW1, layer.dW2, layer.dWr)."""

    def __init__(self, layer: MoELayer):
        import torch
        T, d = layer.dims.T, layer.dims.d
        dev = layer.device
        bf = torch.bfloat16
        self.layer = layer
        self.X = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.dO = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.O = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.dX = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        ev = torch.cuda.Event
        self.inputs_ready = [ev(), ev()]
        self.inputs_free = [ev(), ev()]
        self.fwd_done = [ev(), ev()]
        self.bwd_done = [ev(), ev()]
        self.out_free = [ev(), ev()]
        self.i = 0

    def step(self, Xh, dOh, Oh, Wr, bias, W1, W2, dXh=None):
        """Enqueue one step; Xh, dOh, Oh (and dXh, if given) are pinned host
        tensors [T, d] bf16.  Returns immediately; call finish() before
        reading Oh or dXh.  Without dXh the step's dX stays on the device
        (the buffer of this step's set, self.dX[step % 2])."""
        import torch
        j = self.i & 1
        compute = torch.cuda.current_stream()
        L = self.layer
        with torch.cuda.stream(self.h2d):
            self.h2d.wait_event(self.inputs_free[j])
            self.X[j].copy_(Xh, non_blocking=True)
            self.dO[j].copy_(dOh, non_blocking=True)
            self.inputs_ready[j].record(self.h2d)
        compute.wait_event(self.inputs_ready[j])
        compute.wait_event(self.out_free[j])
        L.route(self.X[j], Wr, bias)
        L.forward(self.X[j], W1, W2, O=self.O[j])
        self.fwd_done[j].record(compute)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.fwd_done[j])
            Oh.copy_(self.O[j], non_blocking=True)
        L.backward(self.dO[j], self.X[j], Wr, W1, W2, dX=self.dX[j])
        self.inputs_free[j].record(compute)
        self.bwd_done[j].record(compute)
        with torch.cuda.stream(self.d2h):
            if dXh is not None:
                self.d2h.wait_event(self.bwd_done[j])
                dXh.copy_(self.dX[j], non_blocking=True)
            self.out_free[j].record(self.d2h)
        self.i += 1

    def finish(self):
        """Make the current stream wait for every copy enqueued so far."""
        import torch
        compute = torch.cuda.current_stream()
        compute.wait_stream(self.h2d)
        compute.wait_stream(self.d2h)
