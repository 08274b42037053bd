"""Python binding of libtm.so with the same call names as include/tm.h.

Argument marshalling only: every step of the forward runs in the library's CUDA
kernels.  PyTorch supplies device memory (outputs and workspaces are allocated
here, by the caller side of the C ABI) and the CUDA stream.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np
import torch

from . import _abi as A

_DT = {torch.float32: A.TM_F32, torch.bfloat16: A.TM_BF16}
_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _p(t: Optional[torch.Tensor]):
    """Device address of a tensor for the C ABI, which reads and writes device memory only and takes
    every tensor dense in row-major order: a host tensor or a strided view is refused here (its
    address would reach a kernel that reads it as something else)."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_cuda:
            raise ValueError(f"libtm takes device tensors; got one on {t.device}")
        if not t.is_contiguous():
            raise ValueError(f"libtm takes contiguous tensors; got strides {t.stride()} for shape {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def lib():
    return A.load()


def shape(B: int, T: int, D: int, H: int, dtype, eps: float = 1e-6) -> A.tm_shape:
    dt = _DT[dtype] if isinstance(dtype, torch.dtype) else (A.TM_BF16 if dtype == "bf16" else A.TM_F32)
    return A.tm_shape(B, T, D, H, dt, eps)


def to_device(arr: np.ndarray, device) -> torch.Tensor:
    """Storage array from tm_synth (uint16 = bf16 bits, float32) -> device tensor of the same bits."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


# ------------------------------------------------------------------ weights
@dataclass
class SubLayer:
    """Device weights of one sub-layer plus its C descriptor (keeps the tensors alive)."""
    is_moe: bool
    banks: int
    width: int
    tensors: Dict[str, torch.Tensor]
    hidden: int = 0
    E: int = 0
    k: int = 0
    hidden_e: int = 0
    hidden_s: int = 0
    alpha: float = 0.0
    gain: Optional[torch.Tensor] = None

    def moe_c(self) -> A.tm_moe_w:
        t = self.tensors
        return A.tm_moe_w(self.banks, self.width, self.E, self.k, self.hidden_e, self.hidden_s, self.alpha,
                          _p(t["w_router"]), _p(t["we_gate"]), _p(t["we_up"]), _p(t["we_down"]),
                          _p(t.get("ws_gate")), _p(t.get("ws_up")), _p(t.get("ws_down")))

    def dense_c(self) -> A.tm_swiglu_w:
        t = self.tensors
        return A.tm_swiglu_w(self.banks, self.width, self.hidden, _p(t["w_gate"]), _p(t["w_up"]), _p(t["w_down"]))

    def c(self) -> A.tm_sublayer:
        s = A.tm_sublayer()
        s.norm_gain = _p(self.gain)
        s.is_moe = 1 if self.is_moe else 0
        if self.is_moe:
            s.moe = self.moe_c()
        else:
            s.dense = self.dense_c()
        return s


@dataclass
class Block:
    mix: SubLayer
    rev: SubLayer

    def c(self) -> A.tm_block:
        return A.tm_block(self.mix.c(), self.rev.c())


def sublayer_from_synth(cfg, layer: int, sub: int, device, down_scale=None, with_gain: bool = False,
                        workers=None) -> SubLayer:
    import tm_synth
    spec = cfg.ffn(sub)
    w = tm_synth.sublayer_weights(cfg, layer, sub, down_scale, workers)
    t = {k: to_device(v, device) for k, v in w.items()}
    g = to_device(tm_synth.gain(cfg, layer, sub), device) if with_gain else None
    if spec.is_moe:
        return SubLayer(True, cfg.banks(sub), cfg.width(sub), t, E=spec.E, k=spec.k, hidden_e=spec.hidden_e,
                        hidden_s=spec.hidden_s, alpha=spec.alpha, gain=g)
    return SubLayer(False, cfg.banks(sub), cfg.width(sub), t, hidden=spec.hidden, gain=g)


def blocks_from_synth(cfg, device, down_scale=None, workers=None) -> List[Block]:
    return [Block(sublayer_from_synth(cfg, l, 0, device, down_scale, workers=workers),
                  sublayer_from_synth(cfg, l, 1, device, down_scale, workers=workers))
            for l in range(cfg.L)]


def config_shape(cfg) -> A.tm_shape:
    return shape(cfg.B, cfg.T, cfg.D, cfg.H, cfg.dtype, cfg.eps)


# ------------------------------------------------------------------ calls
def _ws(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def mix(X: torch.Tensor, H: int, stream=None) -> torch.Tensor:
    B, T, D = X.shape
    out = torch.empty((B, H, T * D // H), dtype=X.dtype, device=X.device)
    sh = shape(B, T, D, H, X.dtype)
    A.check(lib().tm_mix(_p(X), _p(out), ctypes.byref(sh), _s(stream)), "tm_mix")
    return out


def revert(Hm: torch.Tensor, T: int, stream=None) -> torch.Tensor:
    B, H, W = Hm.shape
    D = W * H // T
    out = torch.empty((B, T, D), dtype=Hm.dtype, device=Hm.device)
    sh = shape(B, T, D, H, Hm.dtype)
    A.check(lib().tm_revert(_p(Hm), _p(out), ctypes.byref(sh), _s(stream)), "tm_revert")
    return out


def tokenize_stub(groups: torch.Tensor, w_group: torch.Tensor, w_global: torch.Tensor, D: int, H: int,
                  stream=None) -> torch.Tensor:
    B, G, dg = groups.shape
    out = torch.empty((B, G + 1, D), dtype=groups.dtype, device=groups.device)
    sh = shape(B, G + 1, D, H, groups.dtype)
    A.check(lib().tm_tokenize_stub(_p(groups), _p(w_group), _p(w_global), dg, ctypes.byref(sh), _p(out), _s(stream)),
            "tm_tokenize_stub")
    return out


def route_topk(x: torch.Tensor, layout: int, sh: A.tm_shape, sub: SubLayer, workspace=None, stream=None) -> dict:
    w = sub.moe_c()
    B, banks, k, E = sh.B, sub.banks, sub.k, sub.E
    dev = x.device
    out = {
        "idx": torch.empty((B, banks, k), dtype=torch.int32, device=dev),
        "gate": torch.empty((B, banks, k), dtype=torch.float32, device=dev),
        "gap": torch.empty((B, banks), dtype=torch.float32, device=dev),
        "inv_rms": torch.empty((B, banks), dtype=torch.float32, device=dev),
        "offsets": torch.empty(banks * E + 1, dtype=torch.int32, device=dev),
        "rows": torch.empty(B * banks * k, dtype=torch.int32, device=dev),
        "slot_of": torch.empty((B, banks, k), dtype=torch.int32, device=dev),
    }
    nb = lib().tm_route_workspace_bytes(ctypes.byref(sh), layout, ctypes.byref(w))
    if nb == 0:
        raise A.TMError(A.TM_ERR_INVALID_ARG, "tm_route_workspace_bytes")
    ws = _ws(nb, dev, workspace)
    A.check(lib().tm_route_topk(_p(x), layout, ctypes.byref(sh), _p(sub.gain), ctypes.byref(w), _p(out["idx"]),
                                _p(out["gate"]), _p(out["gap"]), _p(out["inv_rms"]), _p(out["offsets"]),
                                _p(out["rows"]), _p(out["slot_of"]), _p(ws), ws.numel(), _s(stream)), "tm_route_topk")
    return out


def route_topk_noalloc(x: torch.Tensor, layout: int, sh: A.tm_shape, sub: SubLayer, out: dict = None,
                      stream=None) -> dict:
    """tm_route_topk_noalloc: the same routing with the library's fixed scratch array instead of a
    workspace.  `out` may hold preallocated output tensors (the keys route_topk returns), so a
    caller that must not allocate can pass buffers it reserved earlier."""
    w = sub.moe_c()
    B, banks, k, E = sh.B, sub.banks, sub.k, sub.E
    dev = x.device
    if out is None:
        out = {
            "idx": torch.empty((B, banks, k), dtype=torch.int32, device=dev),
            "gate": torch.empty((B, banks, k), dtype=torch.float32, device=dev),
            "gap": torch.empty((B, banks), dtype=torch.float32, device=dev),
            "inv_rms": torch.empty((B, banks), dtype=torch.float32, device=dev),
            "offsets": torch.empty(banks * E + 1, dtype=torch.int32, device=dev),
            "rows": torch.empty(B * banks * k, dtype=torch.int32, device=dev),
            "slot_of": torch.empty((B, banks, k), dtype=torch.int32, device=dev),
        }
    A.check(lib().tm_route_topk_noalloc(_p(x), layout, ctypes.byref(sh), _p(sub.gain), ctypes.byref(w),
                                        _p(out["idx"]), _p(out["gate"]), _p(out.get("gap")), _p(out["inv_rms"]),
                                        _p(out["offsets"]), _p(out["rows"]), _p(out["slot_of"]), _s(stream)),
            "tm_route_topk_noalloc")
    return out


def sublayer_workspace_bytes(sh: A.tm_shape, layout: int, sub: SubLayer) -> int:
    c = sub.c()
    n = lib().tm_sublayer_workspace_bytes(ctypes.byref(sh), layout, ctypes.byref(c))
    if n == 0:
        raise A.TMError(A.TM_ERR_INVALID_ARG, "tm_sublayer_workspace_bytes")
    return n


def _out_like(x: torch.Tensor, layout: int, sh: A.tm_shape, sub: SubLayer) -> torch.Tensor:
    if layout == A.TM_LAYOUT_MIXED:
        return torch.empty((sh.B, sh.T, sh.D), dtype=x.dtype, device=x.device)
    return torch.empty((sh.B, sub.banks, sub.width), dtype=x.dtype, device=x.device)


def pertoken_swiglu(x, residual, layout: int, sh: A.tm_shape, sub: SubLayer, y=None, workspace=None, stream=None):
    y = _out_like(x, layout, sh, sub) if y is None else y
    ws = _ws(sublayer_workspace_bytes(sh, layout, sub), x.device, workspace)
    w = sub.dense_c()
    A.check(lib().tm_pertoken_swiglu(_p(x), _p(residual), layout, ctypes.byref(sh), _p(sub.gain), ctypes.byref(w),
                                     _p(y), _p(ws), ws.numel(), _s(stream)), "tm_pertoken_swiglu")
    return y


def sparse_pertoken_moe(x, residual, layout: int, sh: A.tm_shape, sub: SubLayer, y=None, workspace=None, stream=None):
    y = _out_like(x, layout, sh, sub) if y is None else y
    ws = _ws(sublayer_workspace_bytes(sh, layout, sub), x.device, workspace)
    w = sub.moe_c()
    A.check(lib().tm_sparse_pertoken_moe(_p(x), _p(residual), layout, ctypes.byref(sh), _p(sub.gain),
                                         ctypes.byref(w), _p(y), _p(ws), ws.numel(), _s(stream)),
            "tm_sparse_pertoken_moe")
    return y


def sublayer_forward(x, residual, extra, layout: int, sh: A.tm_shape, sub: SubLayer, y=None, workspace=None,
                     stream=None):
    """tm_sublayer_forward: y = FFN(Norm(x)) + residual + extra for a dense or MoE sub-layer."""
    y = _out_like(x, layout, sh, sub) if y is None else y
    ws = _ws(sublayer_workspace_bytes(sh, layout, sub), x.device, workspace)
    c = sub.c()
    A.check(lib().tm_sublayer_forward(_p(x), _p(residual), _p(extra), layout, ctypes.byref(sh), ctypes.byref(c), _p(y),
                                      _p(ws), ws.numel(), _s(stream)), "tm_sublayer_forward")
    return y


def slice_banks(sub: SubLayer, lo: int, hi: int) -> SubLayer:
    """Banks lo .. hi-1 of a sub-layer (views of its weight tensors, whose leading axis is the bank)."""
    if not (0 <= lo < hi <= sub.banks):
        raise ValueError(f"bank range [{lo}, {hi}) outside [0, {sub.banks})")
    t = {k: v.narrow(0, lo, hi - lo) for k, v in sub.tensors.items()}
    return SubLayer(sub.is_moe, hi - lo, sub.width, t, hidden=sub.hidden, E=sub.E, k=sub.k, hidden_e=sub.hidden_e,
                    hidden_s=sub.hidden_s, alpha=sub.alpha, gain=sub.gain)


def workspace_bytes(sh: A.tm_shape, blocks: Sequence[Block], gap: int = 0) -> int:
    arr = (A.tm_block * len(blocks))(*[b.c() for b in blocks])
    n = lib().tm_workspace_bytes(ctypes.byref(sh), arr, len(blocks), gap)
    if n == 0:
        raise A.TMError(A.TM_ERR_INVALID_ARG, "tm_workspace_bytes")
    return n


def block_forward(X, block: Block, sh: A.tm_shape, Y=None, X_revert=None, workspace=None, stream=None):
    Y = torch.empty_like(X) if Y is None else Y
    c = block.c()
    ws = _ws(workspace_bytes(sh, [block]), X.device, workspace)
    A.check(lib().tm_block_forward(_p(X), ctypes.byref(c), ctypes.byref(sh), _p(Y), _p(X_revert), _p(ws), ws.numel(),
                                   _s(stream)), "tm_block_forward")
    return Y


def stack_step(X, X_skip, block: Block, sh: A.tm_shape, Y=None, X_revert=None, workspace=None, stream=None):
    """tm_stack_step: Y = Block(X) + X_skip (X_skip None: none), one step of the stack forward."""
    Y = torch.empty_like(X) if Y is None else Y
    c = block.c()
    ws = _ws(workspace_bytes(sh, [block]), X.device, workspace)
    A.check(lib().tm_stack_step(_p(X), _p(X_skip), ctypes.byref(c), ctypes.byref(sh), _p(Y), _p(X_revert), _p(ws),
                                ws.numel(), _s(stream)), "tm_stack_step")
    return Y


# Relative chunk sizes of the pipelined end-to-end call: each chunk's host-to-device copy should end
# before the previous chunk's compute does, and its device-to-host copy before the next chunk's
# compute does, so chunks may grow by the ratio of compute to copy time per sample and then shrink,
# leaving only the first copy-in and the last copy-out uncovered; chunks that are too small run
# their grouped GEMMs on nearly empty expert buckets.  Measured on the two MoE stacks (copies 1.7x
# and 4x faster per sample than the forward) against other plans: 1:3:8:3:1 was the fastest on both.
RAMP_CHUNKS = (1, 3, 8, 3, 1)


def chunk_bounds(B: int, chunks) -> List[int]:
    """Sample boundaries [0, ..., B] of the end-to-end call's chunks: `chunks` equal ones (an int) or
    sizes proportional to a sequence of weights; [0, B] (one chunk) when the batch is too small to
    give every chunk two samples."""
    weights = [1] * chunks if isinstance(chunks, int) else list(chunks)
    if len(weights) <= 1 or B < 2 * len(weights):
        return [0, B]
    tot, acc, bounds = float(sum(weights)), 0.0, [0]
    for w in weights:
        acc += w
        bounds.append(int(round(B * acc / tot)))
    return sorted(set(bounds))


def run_host_pipelined(owner, run_rows: Callable, X_host: torch.Tensor, Y_host: torch.Tensor, X_dev: torch.Tensor,
                       Y_dev: torch.Tensor, stream=None, chunks=1) -> torch.Tensor:
    """End to end: pinned host X -> device, forward, device -> pinned host Y; run_rows(a, b, stream)
    runs the forward on samples a .. b-1 of X_dev into Y_dev.

    chunks == 1: all on `stream`.  Otherwise the batch is split along the samples (which are
    independent, so every output is the same bits) and pipelined over three streams: the
    host-to-device copy of chunk i+1 and the device-to-host copy of chunk i-1 run while chunk i
    computes on `stream`.  chunks: a count of equal chunks, or a sequence of relative chunk sizes
    (RAMP_CHUNKS: small first and last chunks, so that little copy time is left uncovered at either
    end, and large ones between, so that few launches run on small batches).  All work of the call
    lies between an event recorded on `stream` at entry and `stream`'s wait for the last copy, so
    events on `stream` around the call time all of it; the next call's work on the same buffers
    starts only after that.  owner keeps the two copy streams between calls."""
    s = torch.cuda.current_stream() if stream is None else stream
    B = X_host.shape[0]
    bounds = chunk_bounds(B, chunks)
    if len(bounds) <= 2:
        with torch.cuda.stream(s):
            X_dev.copy_(X_host, non_blocking=True)
            run_rows(0, B, s)
            Y_host.copy_(Y_dev, non_blocking=True)
        return Y_host
    if not hasattr(owner, "_pipe"):
        owner._pipe = (torch.cuda.Stream(device=X_dev.device), torch.cuda.Stream(device=X_dev.device))
    h2d, d2h = owner._pipe
    n = len(bounds) - 1
    start = torch.cuda.Event()
    start.record(s)
    h2d.wait_event(start)
    done_in, done_out = [], []
    for i in range(n):
        a, b = bounds[i], bounds[i + 1]
        with torch.cuda.stream(h2d):
            X_dev[a:b].copy_(X_host[a:b], non_blocking=True)
            e = torch.cuda.Event()
            e.record(h2d)
            done_in.append(e)
    for i in range(n):
        a, b = bounds[i], bounds[i + 1]
        s.wait_event(done_in[i])
        run_rows(a, b, s)
        e = torch.cuda.Event()
        e.record(s)
        d2h.wait_event(e)
        with torch.cuda.stream(d2h):
            Y_host[a:b].copy_(Y_dev[a:b], non_blocking=True)
            e2 = torch.cuda.Event()
            e2.record(d2h)
            done_out.append(e2)
    s.wait_event(done_out[-1])
    return Y_host


def run_host_steps(owner, run_full: Callable, X_host: torch.Tensor, Y_host: torch.Tensor,
                   X_bufs: Sequence[torch.Tensor], Y_bufs: Sequence[torch.Tensor], steps: int, stream=None) -> torch.Tensor:
    """A stream of `steps` end-to-end steps, as a serving loop runs them: every step copies its batch
    from pinned host memory to the device, runs the forward (run_full(X_dev, Y_dev, stream)) and copies
    the result back, with two device buffers of each so that step i's copy-in and step i-1's copy-out
    run on their own streams while step i-1 and step i compute.  Step i's copy-in waits for step i-2's
    compute (which read the same buffer), step i's compute for step i-2's copy-out.  All of it lies
    between an event recorded on `stream` at entry and `stream`'s wait for the last copy-out, so
    events on `stream` around the call time the whole stream of steps.  Y_host holds the last step's
    result.  owner keeps the two copy streams between calls."""
    s = torch.cuda.current_stream() if stream is None else stream
    if not hasattr(owner, "_pipe"):
        owner._pipe = (torch.cuda.Stream(device=X_bufs[0].device), torch.cuda.Stream(device=X_bufs[0].device))
    h2d, d2h = owner._pipe
    start = torch.cuda.Event()
    start.record(s)
    h2d.wait_event(start)
    d2h.wait_event(start)
    comp, out = [], []
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(comp[i - 2])
            X_bufs[b].copy_(X_host, non_blocking=True)
            e_in = torch.cuda.Event()
            e_in.record(h2d)
        s.wait_event(e_in)
        if i >= 2:
            s.wait_event(out[i - 2])
        run_full(X_bufs[b], Y_bufs[b], s)
        e_c = torch.cuda.Event()
        e_c.record(s)
        comp.append(e_c)
        d2h.wait_event(e_c)
        with torch.cuda.stream(d2h):
            Y_host.copy_(Y_bufs[b], non_blocking=True)
            e_o = torch.cuda.Event()
            e_o.record(d2h)
            out.append(e_o)
    s.wait_event(out[-1])
    return Y_host


class StackRunner:
    """Holds the C block array and a workspace so repeated stack forwards launch with no allocation."""

    def __init__(self, blocks: Sequence[Block], sh: A.tm_shape, gap: int, device):
        self.blocks = list(blocks)
        self.sh = sh
        self.gap = gap
        self.arr = (A.tm_block * len(self.blocks))(*[b.c() for b in self.blocks])
        self.ws = torch.empty(workspace_bytes(sh, self.blocks, gap), dtype=torch.uint8, device=device)

    def __call__(self, X: torch.Tensor, Y: torch.Tensor, stream=None) -> torch.Tensor:
        A.check(lib().tm_stack_forward(_p(X), self.arr, len(self.blocks), self.gap, ctypes.byref(self.sh), _p(Y),
                                       _p(self.ws), self.ws.numel(), _s(stream)), "tm_stack_forward")
        return Y

    def run_host(self, X_host: torch.Tensor, Y_host: torch.Tensor, X_dev: torch.Tensor, Y_dev: torch.Tensor,
                 stream=None, chunks=1) -> torch.Tensor:
        """End to end through tm_stack_forward, pipelined in sample chunks (run_host_pipelined)."""
        def rows(a, b, s):
            sh = A.tm_shape(b - a, self.sh.T, self.sh.D, self.sh.H, self.sh.dtype, self.sh.eps)
            A.check(lib().tm_stack_forward(_p(X_dev[a:b]), self.arr, len(self.blocks), self.gap, ctypes.byref(sh),
                                           _p(Y_dev[a:b]), _p(self.ws), self.ws.numel(), _s(s)), "tm_stack_forward")
        return run_host_pipelined(self, rows, X_host, Y_host, X_dev, Y_dev, stream, chunks)

    def run_host_steps(self, X_host, Y_host, X_bufs, Y_bufs, steps: int, stream=None) -> torch.Tensor:
        """A stream of end-to-end steps, each step's copies overlapping its neighbours' compute."""
        return run_host_steps(self, lambda x, y, s: self(x, y, s), X_host, Y_host, X_bufs, Y_bufs, steps, stream)


def stack_forward(X, blocks: Sequence[Block], gap: int, sh: A.tm_shape, Y=None, stream=None):
    Y = torch.empty_like(X) if Y is None else Y
    return StackRunner(blocks, sh, gap, X.device)(X, Y, stream)


# ------------------------------------------------------------------ scoring head and end-to-end model
def head_forward(X: torch.Tensor, sh: A.tm_shape, w_head: torch.Tensor, stream=None) -> torch.Tensor:
    """tm_head_forward: X [B,T,D] -> logits [B] fp32 (mean over tokens, then w_head [D])."""
    logits = torch.empty((sh.B,), dtype=torch.float32, device=X.device)
    A.check(lib().tm_head_forward(_p(X), ctypes.byref(sh), _p(w_head), _p(logits), _s(stream)), "tm_head_forward")
    return logits


def model_forward(groups, w_group, w_global, blocks: Sequence[Block], gap: int, w_head, sh: A.tm_shape,
                  stream=None) -> torch.Tensor:
    """tm_model_forward: tokenizer -> stack -> head; returns logits [B] fp32."""
    arr = (A.tm_block * len(blocks))(*[b.c() for b in blocks])
    n = lib().tm_model_workspace_bytes(ctypes.byref(sh), arr, len(blocks), gap)
    if n == 0:
        raise A.TMError(A.TM_ERR_INVALID_ARG, "tm_model_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=groups.device)
    logits = torch.empty((sh.B,), dtype=torch.float32, device=groups.device)
    A.check(lib().tm_model_forward(_p(groups), _p(w_group), _p(w_global), groups.shape[-1], arr, len(blocks), gap,
                                   _p(w_head), ctypes.byref(sh), _p(logits), _p(ws), ws.numel(), _s(stream)),
            "tm_model_forward")
    return logits


# ------------------------------------------------------------------ FP8 E4M3 serving path
def quantize_fp8_weights(w: torch.Tensor, gain: Optional[torch.Tensor] = None, stream=None):
    """tm_quantize_fp8_weights: bf16 [groups, rows, cols] matrices -> (E4M3 codes as uint8 of the
    same shape, fp32 scales [groups], one per matrix)."""
    groups, rows, cols = w.shape
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    s = torch.empty((groups,), dtype=torch.float32, device=w.device)
    A.check(lib().tm_quantize_fp8_weights(_p(w), _p(gain), groups, rows, cols, _p(q), _p(s), _s(stream)),
            "tm_quantize_fp8_weights")
    return q, s


def quantize_fp8_act(x: torch.Tensor, layout: int, sh: A.tm_shape, banks: int, width: int, stream=None):
    """tm_quantize_fp8_act: the sub-layer's activation rows -> (codes [B*banks, width] uint8,
    rowscale [B*banks] fp32)."""
    q = torch.empty((sh.B * banks, width), dtype=torch.uint8, device=x.device)
    rs = torch.empty((sh.B * banks,), dtype=torch.float32, device=x.device)
    A.check(lib().tm_quantize_fp8_act(_p(x), layout, ctypes.byref(sh), banks, width, _p(q), _p(rs), _s(stream)),
            "tm_quantize_fp8_act")
    return q, rs


@dataclass
class SubLayer8:
    """A dense sub-layer on the FP8 path: E4M3 gate / up codes with one scale per bank matrix (gain
    folded in) and the bf16 down weights.  Built from a bf16 SubLayer by the library's own quantizer."""
    banks: int
    width: int
    hidden: int
    tensors: Dict[str, torch.Tensor]

    @staticmethod
    def from_bf16(sub: "SubLayer", stream=None) -> "SubLayer8":
        if sub.is_moe:
            raise ValueError("the FP8 path covers dense sub-layers")
        t = sub.tensors
        qg, sg = quantize_fp8_weights(t["w_gate"], sub.gain, stream)
        qu, su = quantize_fp8_weights(t["w_up"], sub.gain, stream)
        return SubLayer8(sub.banks, sub.width, sub.hidden,
                         {"q_gate": qg, "s_gate": sg, "q_up": qu, "s_up": su, "w_down": t["w_down"]})

    def c(self) -> A.tm_swiglu_w8:
        t = self.tensors
        return A.tm_swiglu_w8(self.banks, self.width, self.hidden, _p(t["q_gate"]), _p(t["q_up"]), _p(t["s_gate"]),
                              _p(t["s_up"]), _p(t["w_down"]))


    def sub_c(self) -> A.tm_sublayer8:
        s = A.tm_sublayer8()
        s.is_moe = 0
        s.dense = self.c()
        return s


@dataclass
class MoeSubLayer8:
    """A Sparse-Pertoken MoE sub-layer on the FP8 path: E4M3 gate / up codes of every routed expert
    (one scale per (bank, expert) matrix) and of the shared expert (one per bank), the RMSNorm gain
    folded in by the library's quantizer; the fp32 router, the bf16 down projections and the gain
    (applied by the router) are the bf16 sub-layer's own tensors."""
    banks: int
    width: int
    E: int
    k: int
    hidden_e: int
    hidden_s: int
    alpha: float
    tensors: Dict[str, torch.Tensor]
    gain: Optional[torch.Tensor] = None

    @staticmethod
    def from_bf16(sub: "SubLayer", stream=None) -> "MoeSubLayer8":
        if not sub.is_moe or sub.hidden_s == 0:
            raise ValueError("the FP8 MoE path covers MoE sub-layers with a shared expert")
        t = sub.tensors
        G = sub.banks * sub.E
        qeg, seg = quantize_fp8_weights(t["we_gate"].reshape(G, sub.hidden_e, sub.width), sub.gain, stream)
        qeu, seu = quantize_fp8_weights(t["we_up"].reshape(G, sub.hidden_e, sub.width), sub.gain, stream)
        qsg, ssg = quantize_fp8_weights(t["ws_gate"], sub.gain, stream)
        qsu, ssu = quantize_fp8_weights(t["ws_up"], sub.gain, stream)
        q = {"w_router": t["w_router"], "qe_gate": qeg, "se_gate": seg, "qe_up": qeu, "se_up": seu,
             "we_down": t["we_down"], "qs_gate": qsg, "ss_gate": ssg, "qs_up": qsu, "ss_up": ssu,
             "ws_down": t["ws_down"]}
        return MoeSubLayer8(sub.banks, sub.width, sub.E, sub.k, sub.hidden_e, sub.hidden_s, sub.alpha, q, sub.gain)

    def c(self) -> A.tm_moe_w8:
        t = self.tensors
        return A.tm_moe_w8(self.banks, self.width, self.E, self.k, self.hidden_e, self.hidden_s, self.alpha,
                           _p(t["w_router"]), _p(t["qe_gate"]), _p(t["qe_up"]), _p(t["se_gate"]), _p(t["se_up"]),
                           _p(t["we_down"]), _p(t["qs_gate"]), _p(t["qs_up"]), _p(t["ss_gate"]), _p(t["ss_up"]),
                           _p(t["ws_down"]))

    def sub_c(self) -> A.tm_sublayer8:
        s = A.tm_sublayer8()
        s.norm_gain = _p(self.gain)
        s.is_moe = 1
        s.moe = self.c()
        return s


def sublayer8_from_bf16(sub: "SubLayer", stream=None):
    """The FP8 form of a bf16 sub-layer: MoeSubLayer8 for a MoE bank, SubLayer8 for a dense one."""
    return MoeSubLayer8.from_bf16(sub, stream) if sub.is_moe else SubLayer8.from_bf16(sub, stream)


def sublayer_fp8_workspace_bytes(sh: A.tm_shape, layout: int, sub) -> int:
    c = sub.sub_c()
    n = lib().tm_sublayer_fp8_workspace_bytes(ctypes.byref(sh), layout, ctypes.byref(c))
    if n == 0:
        raise A.TMError(A.TM_ERR_UNSUPPORTED, "tm_sublayer_fp8_workspace_bytes")
    return n


def sublayer_forward_fp8(x, residual, extra, layout: int, sh: A.tm_shape, sub, y=None, workspace=None, stream=None):
    """tm_sublayer_forward_fp8: y = FFN_bank(row) + residual + extra on the FP8 path (sub: SubLayer8 or
    MoeSubLayer8)."""
    if y is None:
        y = (torch.empty((sh.B, sh.T, sh.D), dtype=x.dtype, device=x.device) if layout == A.TM_LAYOUT_MIXED
             else torch.empty((sh.B, sub.banks, sub.width), dtype=x.dtype, device=x.device))
    c = sub.sub_c()
    ws = _ws(sublayer_fp8_workspace_bytes(sh, layout, sub), x.device, workspace)
    A.check(lib().tm_sublayer_forward_fp8(_p(x), _p(residual), _p(extra), layout, ctypes.byref(sh), ctypes.byref(c),
                                          _p(y), _p(ws), ws.numel(), _s(stream)), "tm_sublayer_forward_fp8")
    return y


def sparse_pertoken_moe_fp8(x, residual, layout: int, sh: A.tm_shape, sub: MoeSubLayer8, y=None, workspace=None,
                            stream=None):
    if y is None:
        y = (torch.empty((sh.B, sh.T, sh.D), dtype=x.dtype, device=x.device) if layout == A.TM_LAYOUT_MIXED
             else torch.empty((sh.B, sub.banks, sub.width), dtype=x.dtype, device=x.device))
    w = sub.c()
    ws = _ws(sublayer_fp8_workspace_bytes(sh, layout, sub), x.device, workspace)
    A.check(lib().tm_sparse_pertoken_moe_fp8(_p(x), _p(residual), layout, ctypes.byref(sh), _p(sub.gain),
                                             ctypes.byref(w), _p(y), _p(ws), ws.numel(), _s(stream)),
            "tm_sparse_pertoken_moe_fp8")
    return y


@dataclass
class Block8:
    mix: SubLayer8
    rev: SubLayer8

    @staticmethod
    def from_bf16(block: "Block", stream=None) -> "Block8":
        return Block8(SubLayer8.from_bf16(block.mix, stream), SubLayer8.from_bf16(block.rev, stream))

    def c(self) -> A.tm_block_fp8:
        return A.tm_block_fp8(self.mix.c(), self.rev.c())


def pertoken_swiglu_fp8(x, residual, layout: int, sh: A.tm_shape, sub: SubLayer8, y=None, workspace=None, stream=None):
    if layout == A.TM_LAYOUT_MIXED:
        y = torch.empty((sh.B, sh.T, sh.D), dtype=x.dtype, device=x.device) if y is None else y
    else:
        y = torch.empty((sh.B, sub.banks, sub.width), dtype=x.dtype, device=x.device) if y is None else y
    w = sub.c()
    n = lib().tm_pertoken_swiglu_fp8_workspace_bytes(ctypes.byref(sh), layout, ctypes.byref(w))
    if n == 0:
        raise A.TMError(A.TM_ERR_UNSUPPORTED, "tm_pertoken_swiglu_fp8_workspace_bytes")
    ws = _ws(n, x.device, workspace)
    A.check(lib().tm_pertoken_swiglu_fp8(_p(x), _p(residual), layout, ctypes.byref(sh), ctypes.byref(w), _p(y), _p(ws),
                                         ws.numel(), _s(stream)), "tm_pertoken_swiglu_fp8")
    return y


def block_fp8_workspace_bytes(sh: A.tm_shape, block: Block8) -> int:
    c = block.c()
    n = lib().tm_block_fp8_workspace_bytes(ctypes.byref(sh), ctypes.byref(c))
    if n == 0:
        raise A.TMError(A.TM_ERR_UNSUPPORTED, "tm_block_fp8_workspace_bytes")
    return n


def block_forward_fp8(X, block: Block8, sh: A.tm_shape, Y=None, X_revert=None, workspace=None, stream=None):
    Y = torch.empty_like(X) if Y is None else Y
    c = block.c()
    ws = _ws(block_fp8_workspace_bytes(sh, block), X.device, workspace)
    A.check(lib().tm_block_forward_fp8(_p(X), ctypes.byref(c), ctypes.byref(sh), _p(Y), _p(X_revert), _p(ws),
                                       ws.numel(), _s(stream)), "tm_block_forward_fp8")
    return Y


class Fp8BlockRunner:
    """Consecutive dense blocks on the FP8 path (no inter-residual), with a preallocated workspace
    and ring of intermediate token tensors, so repeated forwards launch with no allocation."""

    def __init__(self, blocks: Sequence[Block8], sh: A.tm_shape, device):
        self.blocks = list(blocks)
        self.sh = sh
        self.cs = [b.c() for b in self.blocks]
        self.ws = torch.empty(max(block_fp8_workspace_bytes(sh, b) for b in self.blocks), dtype=torch.uint8,
                              device=device)
        self.tmp = [torch.empty((sh.B, sh.T, sh.D), dtype=torch.bfloat16, device=device)
                    for _ in range(min(2, len(self.blocks) - 1))]

    def __call__(self, X: torch.Tensor, Y: torch.Tensor, stream=None) -> torch.Tensor:
        cur = X
        for i, c in enumerate(self.cs):
            out = Y if i == len(self.cs) - 1 else self.tmp[i % 2]
            A.check(lib().tm_block_forward_fp8(_p(cur), ctypes.byref(c), ctypes.byref(self.sh), _p(out), None,
                                               _p(self.ws), self.ws.numel(), _s(stream)), "tm_block_forward_fp8")
            cur = out
        return Y

    def run_host(self, X_host, Y_host, X_dev, Y_dev, stream=None):
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            X_dev.copy_(X_host, non_blocking=True)
            self(X_dev, Y_dev, s)
            Y_host.copy_(Y_dev, non_blocking=True)
        return Y_host

    def run_host_steps(self, X_host, Y_host, X_bufs, Y_bufs, steps: int, stream=None) -> torch.Tensor:
        """A stream of end-to-end steps, each step's copies overlapping its neighbours' compute."""
        return run_host_steps(self, lambda x, y, s: self(x, y, s), X_host, Y_host, X_bufs, Y_bufs, steps, stream)


class Fp8StackRunner:
    """A stack on the FP8 path, one tm_sublayer_forward_fp8 call per sub-layer, with the inter-residual
    every `gap` blocks ([digest] 2.3.4: block l adds X_{l-gap} when l % gap == 0, except the last).
    blocks: (mixing, reverting) pairs of SubLayer8 / MoeSubLayer8.  Block l runs
      X_rev = FFN_mix(Mix(X_{l-1})) + Mix(X_{l-1}), stored through Revert (mixed layout, residual X_{l-1});
      X_l   = FFN_rev(X_rev) + X_{l-1} (+ X_{l-gap})                       (row layout)
    with a preallocated workspace and intermediate token tensors, so repeated forwards allocate nothing."""

    def __init__(self, blocks: Sequence, sh: A.tm_shape, gap: int, device):
        self.blocks = list(blocks)
        self.sh = sh
        self.gap = gap
        L = len(self.blocks)
        self.cs = [(m.sub_c(), r.sub_c()) for m, r in self.blocks]
        n = max(max(sublayer_fp8_workspace_bytes(sh, A.TM_LAYOUT_MIXED, m),
                    sublayer_fp8_workspace_bytes(sh, A.TM_LAYOUT_ROWS, r)) for m, r in self.blocks)
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        tok = (sh.B, sh.T, sh.D)
        self.xr = torch.empty(tok, dtype=torch.bfloat16, device=device)
        self.hist = [torch.empty(tok, dtype=torch.bfloat16, device=device) for _ in range(L - 1)]

    def _sub(self, sh, x, resid, extra, layout, c, y, stream):
        A.check(lib().tm_sublayer_forward_fp8(_p(x), _p(resid), _p(extra), layout, ctypes.byref(sh),
                                              ctypes.byref(c), _p(y), _p(self.ws), self.ws.numel(), _s(stream)),
                "tm_sublayer_forward_fp8")

    def rows(self, X: torch.Tensor, Y: torch.Tensor, a: int, b: int, stream=None) -> None:
        """The stack on samples a .. b-1 of X into Y (the intermediates use the same rows)."""
        L = len(self.cs)
        sh = A.tm_shape(b - a, self.sh.T, self.sh.D, self.sh.H, self.sh.dtype, self.sh.eps)
        xs = [X[a:b]] + [h[a:b] for h in self.hist] + [Y[a:b]]
        xr = self.xr[a:b]
        for l in range(1, L + 1):
            cm, cr = self.cs[l - 1]
            self._sub(sh, xs[l - 1], xs[l - 1], None, A.TM_LAYOUT_MIXED, cm, xr, stream)
            skip = xs[l - self.gap] if (self.gap > 0 and l % self.gap == 0 and l < L) else None
            self._sub(sh, xr, xs[l - 1], skip, A.TM_LAYOUT_ROWS, cr, xs[l], stream)

    def __call__(self, X: torch.Tensor, Y: torch.Tensor, stream=None) -> torch.Tensor:
        self.rows(X, Y, 0, X.shape[0], stream)
        return Y

    def run_host(self, X_host, Y_host, X_dev, Y_dev, stream=None, chunks=1):
        """End to end, pipelined in sample chunks (run_host_pipelined)."""
        return run_host_pipelined(self, lambda a, b, s: self.rows(X_dev, Y_dev, a, b, s), X_host, Y_host, X_dev,
                                  Y_dev, stream, chunks)

    def run_host_steps(self, X_host, Y_host, X_bufs, Y_bufs, steps: int, stream=None) -> torch.Tensor:
        """A stream of end-to-end steps, each step's copies overlapping its neighbours' compute."""
        return run_host_steps(self, lambda x, y, s: self(x, y, s), X_host, Y_host, X_bufs, Y_bufs, steps, stream)


def _grads_c(grads: Dict[str, torch.Tensor]) -> A.tm_swiglu_grads:
    return A.tm_swiglu_grads(_p(grads["dw_gate"]), _p(grads["dw_up"]), _p(grads["dw_down"]))


def _grads_like(sub: SubLayer, device) -> Dict[str, torch.Tensor]:
    F, W, nb = sub.hidden, sub.width, sub.banks
    return {"dw_gate": torch.empty((nb, F, W), dtype=torch.bfloat16, device=device),
            "dw_up": torch.empty((nb, F, W), dtype=torch.bfloat16, device=device),
            "dw_down": torch.empty((nb, W, F), dtype=torch.bfloat16, device=device)}


def pertoken_swiglu_backward(x, dy, layout: int, sh: A.tm_shape, sub: SubLayer, dx_add=None, dx=None, grads=None,
                             workspace=None, stream=None):
    """dx and the weight gradients {dw_gate, dw_up, dw_down} of the FFN term of a dense sub-layer
    for the upstream gradient dy (tm_pertoken_swiglu_backward)."""
    dx = torch.empty_like(x) if dx is None else dx
    grads = _grads_like(sub, x.device) if grads is None else grads
    w = sub.dense_c()
    n = lib().tm_pertoken_swiglu_backward_workspace_bytes(ctypes.byref(sh), layout, ctypes.byref(w))
    if n == 0:
        raise A.TMError(A.TM_ERR_UNSUPPORTED, "tm_pertoken_swiglu_backward_workspace_bytes")
    ws = _ws(n, x.device, workspace)
    g = _grads_c(grads)
    A.check(lib().tm_pertoken_swiglu_backward(_p(x), _p(dy), _p(dx_add), layout, ctypes.byref(sh), _p(sub.gain),
                                              ctypes.byref(w), _p(dx), ctypes.byref(g), _p(ws), ws.numel(),
                                              _s(stream)), "tm_pertoken_swiglu_backward")
    return dx, grads


def block_backward_workspace_bytes(sh: A.tm_shape, block: Block) -> int:
    c = block.c()
    n = lib().tm_block_backward_workspace_bytes(ctypes.byref(sh), ctypes.byref(c))
    if n == 0:
        raise A.TMError(A.TM_ERR_UNSUPPORTED, "tm_block_backward_workspace_bytes")
    return n


def block_backward(X, dY, block: Block, sh: A.tm_shape, dX=None, grads=None, workspace=None, stream=None):
    """dX and both sub-layers' weight gradients ({"mix": {...}, "rev": {...}}) of a dense block for
    the gradient dY of its output (tm_block_backward)."""
    dX = torch.empty_like(X) if dX is None else dX
    if grads is None:
        grads = {"mix": _grads_like(block.mix, X.device), "rev": _grads_like(block.rev, X.device)}
    c = block.c()
    ws = _ws(block_backward_workspace_bytes(sh, block), X.device, workspace)
    g = A.tm_block_grads(_grads_c(grads["mix"]), _grads_c(grads["rev"]))
    A.check(lib().tm_block_backward(_p(X), _p(dY), ctypes.byref(c), ctypes.byref(sh), _p(dX), ctypes.byref(g), _p(ws),
                                    ws.numel(), _s(stream)), "tm_block_backward")
    return dX, grads


def stack_backward(X, dY, blocks: Sequence[Block], gap: int, sh: A.tm_shape, dX=None, grads=None, workspace=None,
                   stream=None):
    """dX and every block's weight gradients (a list of {"mix": {...}, "rev": {...}}) of a dense
    stack with the inter-residual every `gap` blocks (tm_stack_backward)."""
    blocks = list(blocks)
    dX = torch.empty_like(X) if dX is None else dX
    if grads is None:
        grads = [{"mix": _grads_like(b.mix, X.device), "rev": _grads_like(b.rev, X.device)} for b in blocks]
    arr = (A.tm_block * len(blocks))(*[b.c() for b in blocks])
    n = lib().tm_stack_backward_workspace_bytes(ctypes.byref(sh), arr, len(blocks), gap)
    if n == 0:
        raise A.TMError(A.TM_ERR_UNSUPPORTED, "tm_stack_backward_workspace_bytes")
    ws = _ws(n, X.device, workspace)
    garr = (A.tm_block_grads * len(blocks))(*[A.tm_block_grads(_grads_c(g["mix"]), _grads_c(g["rev"])) for g in grads])
    A.check(lib().tm_stack_backward(_p(X), _p(dY), arr, len(blocks), gap, ctypes.byref(sh), _p(dX), garr, _p(ws),
                                    ws.numel(), _s(stream)), "tm_stack_backward")
    return dX, grads


class BlockBackwardRunner:
    """Repeated dense-block backward passes with a preallocated workspace and gradient buffers:
    __call__(X, dX) writes dX and the weight gradients for the upstream gradient self.dY."""

    def __init__(self, block: Block, sh: A.tm_shape, dY: torch.Tensor, device):
        self.block = block
        self.sh = sh
        self.c = block.c()
        self.dY = dY
        self.ws = torch.empty(block_backward_workspace_bytes(sh, block), dtype=torch.uint8, device=device)
        self.grads = {"mix": _grads_like(block.mix, device), "rev": _grads_like(block.rev, device)}
        self.gc = A.tm_block_grads(_grads_c(self.grads["mix"]), _grads_c(self.grads["rev"]))

    def __call__(self, X: torch.Tensor, dX: torch.Tensor, stream=None) -> torch.Tensor:
        A.check(lib().tm_block_backward(_p(X), _p(self.dY), ctypes.byref(self.c), ctypes.byref(self.sh), _p(dX),
                                        ctypes.byref(self.gc), _p(self.ws), self.ws.numel(), _s(stream)),
                "tm_block_backward")
        return dX

    def run_host(self, X_host, dX_host, X_dev, dX_dev, dY_host=None, stream=None):
        """End to end on one stream: pinned host X (and dY) -> device, backward, device -> pinned host dX."""
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            X_dev.copy_(X_host, non_blocking=True)
            if dY_host is not None:
                self.dY.copy_(dY_host, non_blocking=True)
            self(X_dev, dX_dev, s)
            dX_host.copy_(dX_dev, non_blocking=True)
        return dX_host


def profile_start() -> None:
    A.check(lib().tm_profile_start(), "tm_profile_start")


def profile_stop(max_entries: int = 64) -> Dict[str, dict]:
    """Per-kernel {launches, total_ms} recorded since profile_start (CUDA events on the launch stream)."""
    arr = (A.tm_kernel_time * max_entries)()
    n = ctypes.c_int(0)
    A.check(lib().tm_profile_stop(arr, max_entries, ctypes.byref(n)), "tm_profile_stop")
    return {arr[i].name.decode(): {"launches": arr[i].launches, "total_ms": arr[i].total_ms} for i in range(n.value)}


def launch_count() -> int:
    return int(lib().tm_launch_count())


def get_device_error(stream=None) -> None:
    A.check(lib().tm_get_device_error(_s(stream)), "device")
