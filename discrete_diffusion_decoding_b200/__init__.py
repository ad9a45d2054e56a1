"""B200-native canvas denoise-sampling stage for uniform-state block diffusion.

Thin Python binding over the C ABI of ``include/dg.h`` (``libdg.so``).  The
functions here only marshal torch tensors into pointers; every step of the path
runs in the library's sm_100a kernels.  There is no CPU or PyTorch fallback: if
the library is missing, importing a function that needs it raises.
"""

import ctypes

import torch

from . import _abi
from ._abi import DgError, DgParams, check, lib

__all__ = ["DgError", "DgParams", "params", "workspace_size", "plan", "temperature", "dg_canvas_init",
           "dg_denoise_step", "dg_stop_check", "dg_stub_hidden", "last_launch_count", "profile_enable",
           "profile_collect", "dg_denoise_stats_noalloc", "dg_debug_set_error", "Workspace", "StepBuffers",
           "decode_batch", "decode_block_ar", "dg_partial_bytes", "dg_denoise_partial", "dg_denoise_merge",
           "dg_debug_set_counter_wait_limit", "dg_quantize_e4m3", "quantize_head_e4m3", "dg_last_sm_clock",
           "dg_tile_head", "tile_head"]


def params(n_canvas, vocab, hidden, **overrides):
    """dg_params with the pages' defaults (48 steps, T 0.8->0.4, bound 0.1, stop 0.005, stability 2)."""
    p = DgParams()
    lib().dg_params_default(ctypes.byref(p), int(n_canvas), int(vocab), int(hidden))
    for k, v in overrides.items():
        if not hasattr(p, k):
            raise KeyError(k)
        setattr(p, k, v)
    return p


def workspace_size(p):
    n = lib().dg_workspace_size(ctypes.byref(p))
    if n == 0:
        raise DgError("dg_workspace_size", _abi.DG_EINVAL, "invalid or unsupported params")
    return n


def plan(p):
    g, ng, sl = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    check("dg_plan", lib().dg_plan(ctypes.byref(p), ctypes.byref(g), ctypes.byref(ng), ctypes.byref(sl)))
    return {"group": g.value, "n_groups": ng.value, "slice": sl.value}


def temperature(p, step):
    return float(lib().dg_temperature(ctypes.byref(p), int(step)))


def profile_enable(max_records):
    """Record CUDA events around the next fused-kernel launches (measurement only)."""
    check("dg_profile_enable", lib().dg_profile_enable(int(max_records)))


def profile_collect():
    """(launches recorded, mean ms, total ms) of the fused kernel since profile_enable."""
    n, mean, tot = ctypes.c_int(), ctypes.c_float(), ctypes.c_float()
    check("dg_profile_collect", lib().dg_profile_collect(ctypes.byref(n), ctypes.byref(mean), ctypes.byref(tot)))
    return n.value, mean.value, tot.value


def last_launch_count():
    return int(lib().dg_last_launch_count())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Workspace:
    """Device workspace for one dg_params (caller-owned memory, as the ABI requires)."""

    def __init__(self, p, device="cuda"):
        self.params = p
        self.nbytes = workspace_size(p)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def dg_canvas_init(p, seeds, tokens, ws, stream=None):
    check("dg_canvas_init", lib().dg_canvas_init(ctypes.byref(p), _ptr(seeds), _ptr(tokens), ws.ptr,
                                                 ws.nbytes, _stream(stream)))


def dg_denoise_step(p, step, h, W, E, seeds, tokens, entropy, argmax, accept, lse, selfcond, ws, stream=None):
    check("dg_denoise_step", lib().dg_denoise_step(
        ctypes.byref(p), int(step), _ptr(h), _ptr(W), _ptr(E), _ptr(seeds), _ptr(tokens), _ptr(entropy),
        _ptr(argmax), _ptr(accept), _ptr(lse), _ptr(selfcond), ws.ptr, ws.nbytes, _stream(stream)))


def dg_stop_check(p, ws, stream=None, want_stable=False):
    """Synchronises the stream; returns (stop_flags list, stable list or None, n_stopped)."""
    C = p.n_canvas
    flags = (ctypes.c_int32 * C)()
    stable = (ctypes.c_int32 * C)() if want_stable else None
    n = ctypes.c_int()
    check("dg_stop_check", lib().dg_stop_check(ctypes.byref(p), ws.ptr, ws.nbytes, flags,
                                               stable if stable is not None else None, ctypes.byref(n),
                                               _stream(stream)))
    return list(flags), (list(stable) if stable is not None else None), n.value


def dg_debug_set_error(p, ws, code, stream=None):
    """Host-side fault injection: write `code` into the workspace's device error word."""
    check("dg_debug_set_error", lib().dg_debug_set_error(ctypes.byref(p), ws.ptr, ws.nbytes, int(code),
                                                         _stream(stream)))


def dg_quantize_e4m3(src, codes, exps, per_row, stream=None):
    """E4M3 codes of a bf16 matrix with power-of-two scales (per row, or one for the tensor)."""
    rows, cols = src.shape
    check("dg_quantize_e4m3", lib().dg_quantize_e4m3(_ptr(src), int(rows), int(cols), int(per_row), _ptr(codes),
                                                     _ptr(exps), _stream(stream)))


def quantize_head_e4m3(W, stream=None):
    """The head as E4M3 codes with one power-of-two scale: returns (codes uint8 [V, d], exponent int).

    Synchronises the stream to read the exponent (a one-time step when a head is loaded).
    """
    codes = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    exps = torch.empty(1, dtype=torch.int32, device=W.device)
    dg_quantize_e4m3(W, codes, exps, 0, stream)
    return codes, int(exps.item())


def dg_last_sm_clock(p, ws, stream=None):
    """SM clock (MHz) at which the last fused pass on this workspace issued its tensor-core work
    (0.0 before the first pass after dg_canvas_init); synchronises the stream."""
    mhz = ctypes.c_float()
    check("dg_last_sm_clock", lib().dg_last_sm_clock(ctypes.byref(p), ws.ptr, ws.nbytes, ctypes.byref(mhz),
                                                     _stream(stream)))
    return float(mhz.value)


def dg_tile_head(src, dst, to_rows, stream=None):
    """Re-order a bf16 [rows, cols] head between row-major (src) and tile-major (dst), or back."""
    rows, cols = src.shape
    check("dg_tile_head", lib().dg_tile_head(_ptr(src), _ptr(dst), int(rows), int(cols), int(to_rows),
                                             _stream(stream)))


def tile_head(W, stream=None):
    """The head in the tile-major layout of params(head_layout=1), as a new [V, d] tensor."""
    out = torch.empty_like(W)
    dg_tile_head(W, out, 0, stream)
    return out


def dg_debug_set_counter_wait_limit(ns):
    """Testing hook: limit the fused kernel's waits on other CTAs' counters to ns (0: the 2 s default)."""
    check("dg_debug_set_counter_wait_limit", lib().dg_debug_set_counter_wait_limit(int(ns)))


def dg_denoise_stats_noalloc(p, step, h, W, E, entropy, argmax, lse, selfcond, stream=None):
    """Fused pass without a caller workspace (scratch lives in the library's fixed device array)."""
    check("dg_denoise_stats_noalloc", lib().dg_denoise_stats_noalloc(
        ctypes.byref(p), int(step), _ptr(h), _ptr(W), _ptr(E), _ptr(entropy), _ptr(argmax), _ptr(lse),
        _ptr(selfcond), _stream(stream)))


def dg_partial_bytes(p):
    """Bytes of one vocabulary shard's partial (statistics + self-conditioning numerator)."""
    n = lib().dg_partial_bytes(ctypes.byref(p))
    if n == 0:
        raise DgError("dg_partial_bytes", _abi.DG_EINVAL, "invalid params")
    return n


def dg_denoise_partial(p, step, v_begin, v_count, h, W_shard, E_shard, seeds, partial, ws, stream=None):
    """Fused pass over vocabulary rows [v_begin, v_begin + v_count) into `partial` (uint8 device buffer)."""
    check("dg_denoise_partial", lib().dg_denoise_partial(
        ctypes.byref(p), int(step), int(v_begin), int(v_count), _ptr(h), _ptr(W_shard), _ptr(E_shard), _ptr(seeds),
        _ptr(partial), ws.ptr, ws.nbytes, _stream(stream)))


def dg_denoise_merge(p, step, n_parts, partials, seeds, tokens, entropy, argmax, accept, lse, selfcond, ws,
                     stream=None):
    """Finish a step from n_parts shard partials laid out back to back in `partials`."""
    check("dg_denoise_merge", lib().dg_denoise_merge(
        ctypes.byref(p), int(step), int(n_parts), _ptr(partials), _ptr(seeds), _ptr(tokens), _ptr(entropy),
        _ptr(argmax), _ptr(accept), _ptr(lse), _ptr(selfcond), ws.ptr, ws.nbytes, _stream(stream)))


def dg_stub_hidden(p, step, gain, noise, seeds, E, tokens, h, ws, stream=None):
    check("dg_stub_hidden", lib().dg_stub_hidden(ctypes.byref(p), int(step), float(gain), float(noise),
                                                 _ptr(seeds), _ptr(E), _ptr(tokens), _ptr(h), ws.ptr, ws.nbytes,
                                                 _stream(stream)))


class StepBuffers:
    """Per-step outputs for N positions (device tensors).

    The per-position results a caller reads every step share one allocation, `packed`
    (entropy float32 [N] | tokens int32 [N] | argmax int32 [N] | accept uint8 [N], 13 N
    bytes), so one device-to-host copy returns them all; the named tensors are views of it.
    """

    def __init__(self, p, device="cuda", selfcond=True):
        N, d = p.n_canvas * p.canvas_len, p.hidden
        self.packed = torch.empty(13 * N, dtype=torch.uint8, device=device)
        self.entropy = self.packed[0:4 * N].view(torch.float32)
        self.tokens = self.packed[4 * N:8 * N].view(torch.int32)
        self.argmax = self.packed[8 * N:12 * N].view(torch.int32)
        self.accept = self.packed[12 * N:13 * N]
        self.lse = torch.empty(N, dtype=torch.float32, device=device)
        self.selfcond = torch.empty((N, d), dtype=torch.float32, device=device) if selfcond else None
        self.h = torch.empty((N, d), dtype=torch.bfloat16, device=device)


def decode_batch(p, W, E, seeds, gain=1.0, noise=0.1, hidden_fn=None, ws=None, bufs=None, on_step=None):
    """Denoise C independent canvases together until each stops or reaches max_steps.

    hidden_fn(tokens, step) -> h fills the denoiser's hidden states; by default the
    benchmark stub (dg_stub_hidden) stands in for the network.  Stopped canvases
    cost nothing in later steps.  Returns (committed [C, 256] int32, stop_step list).
    """
    ws = ws or Workspace(p, W.device)
    bufs = bufs or StepBuffers(p, W.device)
    dg_canvas_init(p, seeds, bufs.tokens, ws)
    C = p.n_canvas
    stop_step = [p.max_steps] * C
    for s in range(1, p.max_steps + 1):
        if hidden_fn is None:
            dg_stub_hidden(p, s, gain, noise, seeds, E, bufs.tokens, bufs.h, ws)
        else:
            bufs.h.copy_(hidden_fn(bufs.tokens, s))
        dg_denoise_step(p, s, bufs.h, W, E, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, bufs.lse,
                        bufs.selfcond, ws)
        if on_step is not None:
            on_step(s, bufs)
        flags, _, n_stopped = dg_stop_check(p, ws)
        for c in range(C):
            if flags[c] and stop_step[c] == p.max_steps and s < p.max_steps:
                stop_step[c] = s
        if n_stopped == C:
            break
    return bufs.argmax.view(C, p.canvas_len).clone(), stop_step


def decode_block_ar(p1, W, E, n_blocks, seed0=0, gain=1.0, noise=0.1, on_step=None):
    """Block-autoregressive decoding: n_blocks canvases of 256 tokens one after another.

    p1 describes one canvas (n_canvas = 1); canvas b uses seed seed0 + b.  The
    committed block of each canvas is appended to the output.  on_step(b, s, bufs),
    if given, sees every step's buffers.  Returns (tokens [n_blocks * 256] int32,
    per-block stop steps).
    """
    ws = Workspace(p1, W.device)
    bufs = StepBuffers(p1, W.device)
    out, steps = [], []
    for b in range(n_blocks):
        seeds = torch.tensor([seed0 + b], dtype=torch.int64, device=W.device)
        cb = None if on_step is None else (lambda s, bf, b=b: on_step(b, s, bf))
        committed, st = decode_batch(p1, W, E, seeds, gain, noise, ws=ws, bufs=bufs, on_step=cb)
        out.append(committed.view(-1))
        steps.append(st[0])
    return torch.cat(out), steps
