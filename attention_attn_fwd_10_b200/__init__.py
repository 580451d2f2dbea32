"""Exact scaled-dot-product attention on B200 (sm_100a): Python binding of libattn.so.

PyTorch is used here only for device memory and streams; every step of the
computation runs in the library's CUDA kernels, reached through the C ABI of
include/attn.h (see ``_abi``).  There is no CPU or PyTorch fallback: on a
machine without the built library or without a CUDA device these functions
raise.

    o, lse = fwd(q, k, v, causal=True)            # q [B,S_q,H_q,D], k/v [B,S_k,H_kv,D] bf16
    o, lse = fwd_split(q, k, v)                   # same result, key range split across CTAs (S_q << S_k)
    dq, dk, dv = bwd(q, k, v, o, lse, do, causal=True)

Inputs may also be CPU tensors: they are copied to the current device, the
kernels run there, and the results are copied back to the host (the
end-to-end path that the benchmark's ``e2e`` figure times).
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _abi
from ._abi import FwdOptions, load, status_string  # noqa: F401

__all__ = ["fwd", "fwd_qk8", "fwd_split", "fwd_split_count", "bwd", "fwd_bwd", "FwdBwdPipeline", "device_status", "set_wait_limit_ns", "exp2_poly_eval", "bwd_workspace_size",
           "load", "status_string"]


def _stream_ptr(stream, device=None) -> int:
    """The raw cudaStream_t of ``stream`` (default: the current stream of
    ``device``), which must belong to ``device``."""
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if device is not None and stream.device != torch.device(device):
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return stream.cuda_stream


def _device_of(*tensors) -> torch.device:
    """The one CUDA device every given tensor lives on (the library's kernels run
    on the current device and must only be handed its memory)."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("every tensor of a call must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices ({dev} and {t.device}): all must be on one device")
    return dev


def _check_tensor(name, t, shape, dtype=torch.bfloat16):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (BSHD, D innermost)")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _shapes(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, S, H, D]")
    B, S_q, H_q, D = q.shape
    S_k, H_kv = k.shape[1], k.shape[2]
    return B, S_q, H_q, S_k, H_kv, D


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
        rescale_threshold: float = 8.0, poly_exp_every: int = 8, rescale_count=None, stream=None,
        persistent: bool = True):
    """Forward attention.  Returns (o bf16 [B,S_q,H_q,D], lse fp32 [B,H_q,S_q]).

    CPU inputs are copied to the current CUDA device and the outputs are
    returned on the CPU.  ``rescale_count``: optional int64 CUDA tensor of one
    element that accumulates the number of O rescales (diagnostic).
    """
    on_host = not q.is_cuda
    if on_host:
        dev = torch.device("cuda", torch.cuda.current_device())
        q, k, v = (t.to(dev, non_blocking=True) for t in (q, k, v))
    B, S_q, H_q, S_k, H_kv, D = _shapes(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check_tensor("q", q, (B, S_q, H_q, D))
    _check_tensor("k", k, (B, S_k, H_kv, D))
    _check_tensor("v", v, (B, S_k, H_kv, D))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H_q, S_q), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, (B, S_q, H_q, D))
    _check_tensor("lse", lse, (B, H_q, S_q), torch.float32)
    dev = _device_of(q, k, v, out, lse, rescale_count)
    opt = FwdOptions(float(rescale_threshold), int(poly_exp_every),
                     rescale_count.data_ptr() if rescale_count is not None else None, int(bool(persistent)))
    with torch.cuda.device(dev):
        code = load().attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  B, H_q, H_kv, S_q, S_k, D, int(bool(causal)), scale, ctypes.byref(opt),
                                  _stream_ptr(stream, dev))
    _abi.check(code, "attn_fwd")
    if on_host:
        return out.cpu(), lse.cpu()
    return out, lse


def fwd_qk8(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
            rescale_threshold: float = 8.0, poly_exp_every: int = 8, stream=None, persistent: bool = True):
    """Forward with 8-bit Q and K (attn_fwd_qk8): q, k torch.float8_e4m3fn, v bf16,
    head dim 128.  Returns (o bf16, lse fp32) of attention over the e4m3 values of
    q and k.  With v torch.float8_e4m3fn as well, both products run on the 8-bit
    path and P is rounded to e4m3 (attn_fwd_qkv8).  Device tensors only."""
    B, S_q, H_q, S_k, H_kv, D = _shapes(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check_tensor("q", q, (B, S_q, H_q, D), torch.float8_e4m3fn)
    _check_tensor("k", k, (B, S_k, H_kv, D), torch.float8_e4m3fn)
    pv8 = v.dtype == torch.float8_e4m3fn
    _check_tensor("v", v, (B, S_k, H_kv, D), torch.float8_e4m3fn if pv8 else torch.bfloat16)
    if out is None:
        out = torch.empty((B, S_q, H_q, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q, S_q), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, (B, S_q, H_q, D))
    _check_tensor("lse", lse, (B, H_q, S_q), torch.float32)
    dev = _device_of(q, k, v, out, lse)
    opt = FwdOptions(float(rescale_threshold), int(poly_exp_every), None, int(bool(persistent)))
    with torch.cuda.device(dev):
        fn = load().attn_fwd_qkv8 if pv8 else load().attn_fwd_qk8
        code = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                  B, H_q, H_kv, S_q, S_k, D, int(bool(causal)), scale, ctypes.byref(opt), _stream_ptr(stream, dev))
    _abi.check(code, "attn_fwd_qkv8" if pv8 else "attn_fwd_qk8")
    return out, lse


def fwd_split_count(B, H_q, H_kv, S_q, S_k, causal: bool = False) -> int:
    """Number of key ranges fwd_split uses by default (attn_fwd_split_count)."""
    return int(load().attn_fwd_split_count(B, H_q, H_kv, S_q, S_k, int(bool(causal))))


def fwd_split(q, k, v, causal: bool = False, scale: float | None = None, num_splits: int = 0, out=None, lse=None,
              workspace=None, stream=None):
    """Split-KV forward (attn_fwd_split): the same (o, lse) as fwd, with the key
    blocks divided among ``num_splits`` ranges (0 = library default) whose partial
    results are merged by the log-sum-exp identity.  q and k may both be
    torch.float8_e4m3fn (attn_fwd_split_qk8, head dim 128).  Device tensors only."""
    B, S_q, H_q, S_k, H_kv, D = _shapes(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    qk8 = q.dtype == torch.float8_e4m3fn
    qk_dtype = torch.float8_e4m3fn if qk8 else torch.bfloat16
    _check_tensor("q", q, (B, S_q, H_q, D), qk_dtype)
    _check_tensor("k", k, (B, S_k, H_kv, D), qk_dtype)
    _check_tensor("v", v, (B, S_k, H_kv, D))
    if out is None:
        out = torch.empty((B, S_q, H_q, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H_q, S_q), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, (B, S_q, H_q, D))
    _check_tensor("lse", lse, (B, H_q, S_q), torch.float32)
    lib = load()
    n = int(num_splits) if num_splits else fwd_split_count(B, H_q, H_kv, S_q, S_k, causal)
    need = int(lib.attn_fwd_split_workspace_size(B, H_q, S_q, D, n)) if n > 1 else 0
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None and workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace holds {workspace.numel() * workspace.element_size()} bytes, needs {need}")
    dev = _device_of(q, k, v, out, lse, workspace)
    fn = lib.attn_fwd_split_qk8 if qk8 else lib.attn_fwd_split
    with torch.cuda.device(dev):
        code = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                  workspace.data_ptr() if workspace is not None else None, B, H_q, H_kv, S_q, S_k, D,
                  int(bool(causal)), scale, n, _stream_ptr(stream, dev))
    _abi.check(code, "attn_fwd_split_qk8" if qk8 else "attn_fwd_split")
    return out, lse


def bwd_workspace_size(B, H_q, S_q, D) -> int:
    return int(load().attn_bwd_workspace_size(B, H_q, S_q, D))


def bwd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, dq=None, dk=None, dv=None,
        workspace=None, stream=None, main_pass_events=None, deterministic: bool = False, cta_mode: int = 0):
    """Backward attention.  Returns (dq, dk, dv) bf16 with the shapes of q, k, v.

    ``main_pass_events``: optional (start, stop) torch.cuda.Event pair recorded
    around the main-pass kernel (diagnostic timing).  ``deterministic``: add the
    dQ parts of each query block in key-tile order (bitwise reproducible dQ).
    ``cta_mode``: 0 = the faster kernel of each mode (CTA pairs for the
    deterministic backward at head dim 128, else one CTA per key tile), 1 = one
    CTA per key tile, 2 = CTA pairs whose tensor cores execute each MMA together
    (head dim 128)."""
    on_host = not q.is_cuda
    if on_host:
        dev = torch.device("cuda", torch.cuda.current_device())
        q, k, v, o, lse, do = (t.to(dev, non_blocking=True) for t in (q, k, v, o, lse, do))
    B, S_q, H_q, S_k, H_kv, D = _shapes(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check_tensor("q", q, (B, S_q, H_q, D))
    _check_tensor("k", k, (B, S_k, H_kv, D))
    _check_tensor("v", v, (B, S_k, H_kv, D))
    _check_tensor("o", o, (B, S_q, H_q, D))
    _check_tensor("lse", lse, (B, H_q, S_q), torch.float32)
    _check_tensor("do", do, (B, S_q, H_q, D))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for n, t, shp in (("dq", dq, q.shape), ("dk", dk, k.shape), ("dv", dv, v.shape)):
        _check_tensor(n, t, shp)
    need = bwd_workspace_size(B, H_q, S_q, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < need or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of at least {need} bytes")
    dev = _device_of(q, k, v, o, lse, do, dq, dk, dv, workspace)
    opt = None
    with torch.cuda.device(dev):
        if main_pass_events is not None or deterministic or cta_mode:
            ev = (None, None)
            if main_pass_events is not None:
                s = torch.cuda.current_stream(dev) if stream is None else stream
                for e in main_pass_events:
                    if e.cuda_event == 0:  # torch creates the CUDA event lazily, on its first record
                        e.record(s)
                ev = (main_pass_events[0].cuda_event, main_pass_events[1].cuda_event)
            opt = ctypes.byref(_abi.BwdOptions(ev[0], ev[1], int(bool(deterministic)), int(cta_mode)))
        code = load().attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                  B, H_q, H_kv, S_q, S_k, D, int(bool(causal)), scale, opt,
                                  _stream_ptr(stream, dev))
    _abi.check(code, "attn_bwd")
    if on_host:
        return dq.cpu(), dk.cpu(), dv.cpu()
    return dq, dk, dv


def fwd_bwd(q, k, v, do, causal: bool = False, scale: float | None = None, host_out: dict | None = None,
            stream=None):
    """One training step of attention from host buffers: copy q, k, v, dO to the
    current device, run the forward and the backward there, and copy o, lse,
    dq, dk, dv back into ``host_out`` (pinned CPU tensors, allocated if None).
    Returns the dict of host results."""
    dev = torch.device("cuda", torch.cuda.current_device())
    qd, kd, vd, dod = (t.to(dev, non_blocking=True) for t in (q, k, v, do))
    o, lse = fwd(qd, kd, vd, causal=causal, scale=scale, stream=stream)
    dq, dk, dv = bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale, stream=stream)
    if host_out is None:
        host_out = {}
    res = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    for name, t in res.items():
        if name in host_out:
            host_out[name].copy_(t, non_blocking=True)
        else:
            host_out[name] = t.to("cpu")
    torch.cuda.current_stream().synchronize()
    return host_out


class FwdBwdPipeline:
    """Attention training steps (forward + backward) from pinned host buffers,
    with the copies of one step overlapping the kernels of its neighbours.

    Three streams: the inputs of a step (q, k, v, dO) go up on one copy stream,
    its kernels run on a compute stream, and its results (o, lse, dq, dk, dv)
    come down on a second copy stream.  ``depth`` sets of device buffers rotate
    between steps, so step k+1 uploads while step k computes and step k-1
    downloads.  Every step still moves all its inputs up and all its results
    down; only the order of the work changes.

        pipe = FwdBwdPipeline(B, S_q, S_k, H_q, H_kv, D, causal=True)
        for hq, hk, hv, hdo, out in steps:      # pinned CPU tensors; out: dict of pinned tensors
            pipe.submit(hq, hk, hv, hdo, out)
        pipe.synchronize()                        # every submitted step's results are in `out`
    """

    def __init__(self, B, S_q, S_k, H_q, H_kv, D, causal: bool = False, scale: float | None = None,
                 depth: int = 2, device=None):
        self.dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.causal = bool(causal)
        self.scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
        self.up, self.compute, self.down = (torch.cuda.Stream(self.dev) for _ in range(3))
        bf, dev = torch.bfloat16, self.dev
        ws = bwd_workspace_size(B, H_q, S_q, D)
        self.sets = []
        for _ in range(max(1, int(depth))):
            self.sets.append({
                "q": torch.empty((B, S_q, H_q, D), dtype=bf, device=dev),
                "k": torch.empty((B, S_k, H_kv, D), dtype=bf, device=dev),
                "v": torch.empty((B, S_k, H_kv, D), dtype=bf, device=dev),
                "do": torch.empty((B, S_q, H_q, D), dtype=bf, device=dev),
                "o": torch.empty((B, S_q, H_q, D), dtype=bf, device=dev),
                "lse": torch.empty((B, H_q, S_q), dtype=torch.float32, device=dev),
                "dq": torch.empty((B, S_q, H_q, D), dtype=bf, device=dev),
                "dk": torch.empty((B, S_k, H_kv, D), dtype=bf, device=dev),
                "dv": torch.empty((B, S_k, H_kv, D), dtype=bf, device=dev),
                "ws": torch.empty(ws, dtype=torch.uint8, device=dev),
                "uploaded": torch.cuda.Event(), "computed": torch.cuda.Event(), "downloaded": None,
            })
        self.n = 0

    def submit(self, q, k, v, do, host_out: dict) -> None:
        """Enqueue one step.  q, k, v, do: pinned CPU tensors; host_out: dict with
        pinned CPU tensors "o", "lse", "dq", "dk", "dv" that receive the results
        (valid after synchronize(), or once a later step's submit returned and
        the caller synchronised).  Neither may be modified until then."""
        s = self.sets[self.n % len(self.sets)]
        self.n += 1
        if s["downloaded"] is not None:  # this set's previous results must be down first
            self.up.wait_event(s["downloaded"])
        with torch.cuda.stream(self.up):
            for name, t in (("q", q), ("k", k), ("v", v), ("do", do)):
                s[name].copy_(t, non_blocking=True)
            s["uploaded"].record(self.up)
        self.compute.wait_event(s["uploaded"])
        fwd(s["q"], s["k"], s["v"], causal=self.causal, scale=self.scale, out=s["o"], lse=s["lse"],
            stream=self.compute)
        bwd(s["q"], s["k"], s["v"], s["o"], s["lse"], s["do"], causal=self.causal, scale=self.scale,
            dq=s["dq"], dk=s["dk"], dv=s["dv"], workspace=s["ws"], stream=self.compute)
        s["computed"].record(self.compute)
        self.down.wait_event(s["computed"])
        with torch.cuda.stream(self.down):
            for name in ("o", "lse", "dq", "dk", "dv"):
                host_out[name].copy_(s[name], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.down)
            s["downloaded"] = ev

    def synchronize(self) -> None:
        for st in (self.up, self.compute, self.down):
            st.synchronize()


def device_status(stream=None) -> int:
    """Read and clear the current device's status word after the stream's work;
    returns the code (0 = OK).  The word is shared by every stream of the device."""
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(load().attn_device_status(_stream_ptr(stream, dev)))


def set_wait_limit_ns(ns: int) -> None:
    load().attn_set_wait_limit_ns(int(ns))


def exp2_poly_eval(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The kernels' FMA-pipe cubic 2^x evaluated on a CUDA fp32 tensor (diagnostic)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        _abi.check(load().attn_exp2_poly_eval(x.data_ptr(), y.data_ptr(), x.numel(), _stream_ptr(stream, x.device)),
                   "attn_exp2_poly_eval")
    return y
