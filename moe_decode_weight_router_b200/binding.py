"""Python binding of libmoe_decode.so: the C-ABI entry points under the same names.

Argument marshalling only -- torch tensors in, raw device pointers and sizes out
to the library; every step of the computation runs in the library's CUDA
kernels.  torch provides device memory and streams.  A missing library raises;
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import torch

from . import _abi


class MoeError(RuntimeError):
    def __init__(self, name: str, status: int):
        lib = _abi.load()
        msg = lib.moe_status_string(status).decode()
        if status == 6:
            msg += f" (cudaError {lib.moe_last_cuda_error()})"
        super().__init__(f"{name}: {msg}")
        self.status = status


def _lib():
    return _abi.load()


def _check(name: str, status: int):
    if status != 0:
        raise MoeError(name, status)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _dev_bf16(t: torch.Tensor, name: str):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
        raise TypeError(f"{name}: expected a contiguous CUDA bfloat16 tensor")


def abi_version() -> int:
    return _lib().moe_abi_version()


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    """Device-side status word of the last call on ``ws`` (0 = OK, 7 = timeout)."""
    return _lib().moe_workspace_status(_ptr(ws), _stream(stream))


def moe_selfcheck(device=None, stream=None):
    """Runs the library's start-up self-check on ``device`` (default: the current CUDA
    device).  Returns (status, failed_check, max_rel_l2); status 0 means every check
    passed, 8 (MOE_ERR_SELFCHECK) that check ``failed_check`` gave a wrong result."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    ws = _ws(_lib().moe_selfcheck_workspace_bytes(), dev)
    fail, rel = ctypes.c_int(0), ctypes.c_float(0.0)
    st = _lib().moe_selfcheck(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(fail), ctypes.byref(rel))
    return st, fail.value, rel.value


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------
def moe_route_workspace_bytes(M: int, E: int) -> int:
    return _lib().moe_route_workspace_bytes(M, E)


def moe_route(x: torch.Tensor, w_router: torch.Tensor, top_k: int, *, logits: bool = False, ws=None,
              out=None, stream=None):
    """Router top-k of bf16 tokens x [M,H] against bf16 w_router [E,H].

    Returns (ids int32 [M,k], weights fp32 [M,k], logits fp32 [M,E] or None)."""
    _dev_bf16(x, "x")
    _dev_bf16(w_router, "w_router")
    M, H = x.shape
    E = w_router.shape[0]
    dev = x.device
    if out is None:
        ids = torch.empty((M, top_k), dtype=torch.int32, device=dev)
        w = torch.empty((M, top_k), dtype=torch.float32, device=dev)
        lg = torch.empty((M, E), dtype=torch.float32, device=dev) if logits else None
    else:
        ids, w, lg = out
    if ws is None:
        ws = _ws(moe_route_workspace_bytes(M, E), dev)
    _check("moe_route", _lib().moe_route(_ptr(x), M, H, _ptr(w_router), E, top_k, _ptr(ids), _ptr(w),
                                          _ptr(lg), _ptr(ws), ws.numel(), _stream(stream)))
    return ids, w, lg


# ---------------------------------------------------------------------------
# Experts
# ---------------------------------------------------------------------------
def moe_experts_workspace_bytes(M, H, I, E, top_k, Is) -> int:
    return _lib().moe_experts_workspace_bytes(M, H, I, E, top_k, Is)


def moe_mxfp4_experts(x, topk_ids, topk_w, w13c, w13s, w2c, w2s, sw13=None, sw2=None, *, ws=None, y=None,
                      stream=None):
    """One MoE layer y [M,H] fp32 for bf16 x [M,H] under the given routing."""
    _dev_bf16(x, "x")
    M, H = x.shape
    E, twoI, _ = w13c.shape
    I = twoI // 2
    k = topk_ids.shape[1]
    Is = sw13.shape[0] // 2 if sw13 is not None else 0
    dev = x.device
    if y is None:
        y = torch.empty((M, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _ws(moe_experts_workspace_bytes(M, H, I, E, k, Is), dev)
    _check("moe_mxfp4_experts", _lib().moe_mxfp4_experts(
        _ptr(x), M, H, I, E, k, _ptr(topk_ids), _ptr(topk_w), _ptr(w13c), _ptr(w13s), _ptr(w2c), _ptr(w2s),
        _ptr(sw13), _ptr(sw2), Is, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y


# ---------------------------------------------------------------------------
# prefill chunk (tcgen05 block-scaled path)
# ---------------------------------------------------------------------------
def moe_prefill_workspace_bytes(M, H, I, E, top_k, Is) -> int:
    return _lib().moe_prefill_workspace_bytes(M, H, I, E, top_k, Is)


def moe_prefill_layer(x, wr, w13c, w13s, w2c, w2s, sw13=None, sw2=None, *, top_k, ws=None, y=None,
                      want_routing: bool = True, want_logits: bool = False, stream=None):
    """One MoE layer over a prefill chunk: bf16 x [M,H] -> (y fp32 [M,H], ids [M,k], w [M,k], logits [M,E]).

    Routing, shared expert and routed experts all run in this call (MXFP8
    activations for the routed experts); ids/w/logits are None unless asked for."""
    _dev_bf16(x, "x")
    M, H = x.shape
    E, twoI, _ = w13c.shape
    I = twoI // 2
    Is = sw13.shape[0] // 2 if sw13 is not None else 0
    dev = x.device
    if y is None:
        y = torch.empty((M, H), dtype=torch.float32, device=dev)
    ids = torch.empty((M, top_k), dtype=torch.int32, device=dev) if want_routing else None
    w = torch.empty((M, top_k), dtype=torch.float32, device=dev) if want_routing else None
    lg = torch.empty((M, E), dtype=torch.float32, device=dev) if want_logits else None
    if ws is None:
        ws = _ws(moe_prefill_workspace_bytes(M, H, I, E, top_k, Is), dev)
    _check("moe_prefill_layer", _lib().moe_prefill_layer(
        _ptr(x), M, H, I, E, top_k, _ptr(wr), _ptr(w13c), _ptr(w13s), _ptr(w2c), _ptr(w2s), _ptr(sw13), _ptr(sw2),
        Is, _ptr(ids), _ptr(w), _ptr(lg), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y, ids, w, lg


def moe_mxfp8_quantize(v, *, stream=None):
    """fp32 [M,K] -> (e4m3 codes uint8 [M,K], E8M0 scales uint8 [M,K/32])."""
    if v.dtype != torch.float32 or not v.is_cuda or not v.is_contiguous():
        raise TypeError("v: expected a contiguous CUDA float32 tensor")
    M, K = v.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=v.device)
    s = torch.empty((M, K // 32), dtype=torch.uint8, device=v.device)
    _check("moe_mxfp8_quantize", _lib().moe_mxfp8_quantize(_ptr(v), M, K, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


# ---------------------------------------------------------------------------
# LM head
# ---------------------------------------------------------------------------
def lm_head_fp8_quantize(w: torch.Tensor, *, out=None, stream=None):
    """BF16 [V,H] -> (e4m3 codes uint8 [V,H], fp32 row scales [V])."""
    _dev_bf16(w, "w")
    V, H = w.shape
    if out is None:
        q = torch.empty((V, H), dtype=torch.uint8, device=w.device)
        s = torch.empty((V,), dtype=torch.float32, device=w.device)
    else:
        q, s = out
    _check("lm_head_fp8_quantize", _lib().lm_head_fp8_quantize(_ptr(w), V, H, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def lm_head_workspace_bytes(M, V, H) -> int:
    return _lib().lm_head_workspace_bytes(M, V, H)


def lm_head_fp8_gemv(x, q, s, *, want_logits: bool = True, ws=None, out=None, stream=None):
    """Returns (logits fp32 [M,V] or None, argmax int32 [M])."""
    _dev_bf16(x, "x")
    M, H = x.shape
    V = q.shape[0]
    dev = x.device
    if out is None:
        logits = torch.empty((M, V), dtype=torch.float32, device=dev) if want_logits else None
        am = torch.empty((M,), dtype=torch.int32, device=dev)
    else:
        logits, am = out
    if ws is None:
        ws = _ws(lm_head_workspace_bytes(M, V, H), dev)
    _check("lm_head_fp8_gemv", _lib().lm_head_fp8_gemv(_ptr(x), M, V, H, _ptr(q), _ptr(s), _ptr(logits), _ptr(am),
                                                        _ptr(ws), ws.numel(), _stream(stream)))
    return logits, am


def lm_head_fp8_verify(x, q, s, drafts, *, want_logits: bool = False, ws=None, stream=None):
    """Verify window: (logits or None, argmax int32 [M], accept int32 [1+M]) -- accept[0]
    is the accepted count, accept[1:1+count] the accepted tokens."""
    _dev_bf16(x, "x")
    M, H = x.shape
    V = q.shape[0]
    dev = x.device
    logits = torch.empty((M, V), dtype=torch.float32, device=dev) if want_logits else None
    am = torch.empty((M,), dtype=torch.int32, device=dev)
    acc = torch.empty((1 + M,), dtype=torch.int32, device=dev)
    d = drafts.to(device=dev, dtype=torch.int32).contiguous()
    if ws is None:
        ws = _ws(lm_head_workspace_bytes(M, V, H), dev)
    _check("lm_head_fp8_verify", _lib().lm_head_fp8_verify(_ptr(x), M, V, H, _ptr(q), _ptr(s), _ptr(d), _ptr(logits),
                                                            _ptr(am), _ptr(acc), _ptr(ws), ws.numel(), _stream(stream)))
    return logits, am, acc


def lm_head_bf16_gemv(x, w, *, want_logits: bool = True, ws=None, out=None, stream=None):
    """BF16-weight head: (logits fp32 [M,V] or None, argmax int32 [M])."""
    _dev_bf16(x, "x")
    _dev_bf16(w, "w")
    M, H = x.shape
    V = w.shape[0]
    dev = x.device
    if out is None:
        logits = torch.empty((M, V), dtype=torch.float32, device=dev) if want_logits else None
        am = torch.empty((M,), dtype=torch.int32, device=dev)
    else:
        logits, am = out
    if ws is None:
        ws = _ws(lm_head_workspace_bytes(M, V, H), dev)
    _check("lm_head_bf16_gemv", _lib().lm_head_bf16_gemv(_ptr(x), M, V, H, _ptr(w), _ptr(logits), _ptr(am), _ptr(ws),
                                                          ws.numel(), _stream(stream)))
    return logits, am


def moe_sample(logits, u, *, temperature: float, top_k: int, top_p: float, stream=None):
    """One sampled token id per row of fp32 logits [M,V]; u [M] fp32 uniform draws."""
    if logits.dtype != torch.float32 or not logits.is_cuda or not logits.is_contiguous():
        raise TypeError("logits: expected a contiguous CUDA float32 tensor")
    M, V = logits.shape
    uu = u.to(device=logits.device, dtype=torch.float32).contiguous()
    ids = torch.empty((M,), dtype=torch.int32, device=logits.device)
    _check("moe_sample", _lib().moe_sample(_ptr(logits), M, V, float(temperature), int(top_k), float(top_p), _ptr(uu),
                                           _ptr(ids), _stream(stream)))
    return ids


def lm_head_fp8_gemv_noalloc(x, q, s, *, want_logits: bool = True, out=None, stream=None):
    """As lm_head_fp8_gemv, through the entry point that takes no workspace (the
    library's static per-device control block; calls must not overlap)."""
    _dev_bf16(x, "x")
    M, H = x.shape
    V = q.shape[0]
    dev = x.device
    if out is None:
        logits = torch.empty((M, V), dtype=torch.float32, device=dev) if want_logits else None
        am = torch.empty((M,), dtype=torch.int32, device=dev)
    else:
        logits, am = out
    _check("lm_head_fp8_gemv_noalloc", _lib().lm_head_fp8_gemv_noalloc(
        _ptr(x), M, V, H, _ptr(q), _ptr(s), _ptr(logits), _ptr(am), _stream(stream)))
    return logits, am


# ---------------------------------------------------------------------------
# Whole decode step
# ---------------------------------------------------------------------------
@dataclass
class DecodeModel:
    """Host-side model descriptor (device tensors + format tags) for decode_step."""
    layers: list            # dicts with wr, w13c, w13s, w2c, w2s, sw13, sw2 (torch CUDA tensors)
    lm_q: torch.Tensor      # [V,H] uint8 e4m3
    lm_s: torch.Tensor      # [V] fp32
    top_k: int
    rms_eps: float = 1e-6
    lm_fmt: int = _abi.FMT_E4M3
    step_path: int = _abi.STEP_AUTO
    _keep: list = field(default_factory=list, repr=False)

    def cstruct(self) -> _abi.Model:
        L0 = self.layers[0]
        E, H = L0["wr"].shape
        I = L0["w13c"].shape[1] // 2
        Is = L0["sw13"].shape[0] // 2 if L0.get("sw13") is not None else 0
        arr = (_abi.Layer * len(self.layers))()
        for i, L in enumerate(self.layers):
            arr[i].router = _abi.Buf(L["wr"].data_ptr(), _abi.FMT_BF16)
            arr[i].w13_codes = _abi.Buf(L["w13c"].data_ptr(), _abi.FMT_MXFP4_CODES)
            arr[i].w13_scales = _abi.Buf(L["w13s"].data_ptr(), _abi.FMT_E8M0_SCALES)
            arr[i].w2_codes = _abi.Buf(L["w2c"].data_ptr(), _abi.FMT_MXFP4_CODES)
            arr[i].w2_scales = _abi.Buf(L["w2s"].data_ptr(), _abi.FMT_E8M0_SCALES)
            if Is:
                arr[i].shared_w13 = _abi.Buf(L["sw13"].data_ptr(), _abi.FMT_BF16)
                arr[i].shared_w2 = _abi.Buf(L["sw2"].data_ptr(), _abi.FMT_BF16)
        m = _abi.Model(len(self.layers), H, I, E, self.top_k, Is, self.lm_q.shape[0], self.rms_eps,
                       ctypes.cast(arr, ctypes.POINTER(_abi.Layer)),
                       _abi.Buf(self.lm_q.data_ptr(), self.lm_fmt), _abi.Buf(self.lm_s.data_ptr(), _abi.FMT_F32),
                       self.step_path)
        self._keep = [arr, m]
        return m


def decode_step_launch_names(model: DecodeModel, M: int) -> list:
    """Names of the kernels one decode_step launches, in launch order."""
    m = model.cstruct()
    n = _lib().decode_step_launch_names(ctypes.byref(m), M, None, 0)
    if n < 0:
        raise MoeError("decode_step_launch_names", 1)
    arr = (ctypes.c_char_p * n)()
    _lib().decode_step_launch_names(ctypes.byref(m), M, arr, n)
    return [a.decode() for a in arr]


def decode_step_workspace_bytes(model: DecodeModel, M: int) -> int:
    m = model.cstruct()
    return _lib().decode_step_workspace_bytes(ctypes.byref(m), M)


def _event_array(events):
    if not events:
        return None, 0
    for e in events:
        if not e.cuda_event:  # torch creates the CUDA event lazily, on its first record
            e.record()
    torch.cuda.current_stream().synchronize()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    return arr, len(events)


def decode_step(model: DecodeModel, x: torch.Tensor, *, want_logits: bool = True, trace: bool = False, ws=None,
                out=None, stream=None, events=None, timeline=None, wait_limit_ns: int = 0, hold_layer=None):
    """One decode step.  Returns dict(logits, argmax[, trace tensors]).

    ``events``: optional list of torch.cuda.Event(enable_timing=True), recorded in
    pairs around each kernel launch of the step (see moe_trace_t).  ``wait_limit_ns`` and
    ``hold_layer`` exercise the timeout path (a layer whose residual is never published,
    and a short limit on every bounded device wait): testing only."""
    _dev_bf16(x, "x")
    M, H = x.shape
    dev = x.device
    m = model.cstruct()
    V = model.lm_q.shape[0]
    L = len(model.layers)
    k = model.top_k
    if out is None:
        logits = torch.empty((M, V), dtype=torch.float32, device=dev) if want_logits else None
        am = torch.empty((M,), dtype=torch.int32, device=dev)
    else:
        logits, am = out
    res = {"logits": logits, "argmax": am}
    tr = None
    evs, nev = _event_array(events)
    if trace:
        res["x_trace"] = torch.empty((L + 1, M, H), dtype=torch.bfloat16, device=dev)
        res["h_trace"] = torch.empty((L + 1, M, H), dtype=torch.float32, device=dev)
        res["ids_trace"] = torch.empty((L, M, k), dtype=torch.int32, device=dev)
        res["w_trace"] = torch.empty((L, M, k), dtype=torch.float32, device=dev)
        tr = _abi.Trace(res["x_trace"].data_ptr(), res["h_trace"].data_ptr(), res["ids_trace"].data_ptr(),
                        res["w_trace"].data_ptr(), evs, nev)
    elif evs is not None:
        tr = _abi.Trace(None, None, None, None, evs, nev)
    if timeline is not None or wait_limit_ns or hold_layer is not None:
        if tr is None:
            tr = _abi.Trace(None, None, None, None, None, 0)
        if timeline is not None:
            tr.timeline = timeline.data_ptr()
        tr.wait_limit_ns = int(wait_limit_ns)
        tr.hold_layer = 0 if hold_layer is None else int(hold_layer) + 1
    if ws is None:
        ws = _ws(_lib().decode_step_workspace_bytes(ctypes.byref(m), M), dev)
    _check("decode_step", _lib().decode_step(ctypes.byref(m), _ptr(x), M, _ptr(logits), _ptr(am),
                                              ctypes.byref(tr) if tr is not None else None, _ptr(ws), ws.numel(),
                                              _stream(stream)))
    res["ws"] = ws
    return res


class DecodeGraph:
    """decode_step captured once as a CUDA graph bound to fixed x / logits / argmax buffers."""

    def __init__(self, model: DecodeModel, x: torch.Tensor, logits, argmax, ws, events=None, trace=None):
        """``trace``: optional dict with x_trace/h_trace/ids_trace/w_trace device tensors
        (shapes as decode_step(trace=True) returns) that every replay fills."""
        self.model, self.x, self.logits, self.argmax, self.ws = model, x, logits, argmax, ws
        self._m = model.cstruct()
        self._evs, nev = _event_array(events)
        self.events, self.trace = events, trace
        tr = None
        if trace is not None or self._evs is not None:
            t = trace or {}
            tr = _abi.Trace(*(t[n].data_ptr() if n in t else None for n in ("x_trace", "h_trace", "ids_trace",
                                                                              "w_trace")), self._evs, nev)
        h = ctypes.c_void_p()
        _check("decode_step_graph_create", _lib().decode_step_graph_create(
            ctypes.byref(self._m), _ptr(x), x.shape[0], _ptr(logits), _ptr(argmax),
            ctypes.byref(tr) if tr is not None else None, _ptr(ws), ws.numel(), ctypes.byref(h)))
        self._h = h

    def launch(self, stream=None):
        _check("decode_step_graph_launch", _lib().decode_step_graph_launch(self._h, _stream(stream)))

    def close(self):
        if self._h:
            _lib().decode_step_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
