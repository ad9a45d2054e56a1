"""Vocabulary-parallel split of one denoising step (one process per GPU).

Rank r of a group of G holds the vocabulary rows [v_r, v_{r+1}) of W and E.  A step
is: the fused pass over the shard (dg_denoise_partial: the shard's log-sum-exp
statistics, argmax, sampled key and self-conditioning numerator per position), one
all-gather of those partials over the group, and the merge on every rank
(dg_denoise_merge: entropy, argmax, log-sum-exp, self-conditioning, accept /
re-noise and the stop reduction).  Every rank merges the same partials, so the
canvases and stop flags stay identical without further exchange; the re-noise draws
are keyed on (seed, step, position) and need none.

The pages describe no multi-device scheme; this split follows from the exact merge
of log-sum-exp statistics over disjoint vocabulary ranges.  This module only moves
buffers between ranks (torch.distributed); every step of the computation runs in
the library's kernels.
"""

import torch
import torch.distributed as tdist

from . import Workspace, dg_canvas_init, dg_denoise_merge, dg_denoise_partial, dg_partial_bytes

ALIGN = 256   # shard boundaries are multiples of the fused kernel's vocabulary tile


def shard_bounds(vocab, world, rank, align=ALIGN):
    """Contiguous rows [v0, v1) of shard `rank` of `world`: multiples of `align`, sizes within one unit."""
    if vocab % align or vocab // align < world:
        raise ValueError(f"vocab {vocab} does not split into {world} shards of multiples of {align}")
    units = vocab // align
    return units * rank // world * align, units * (rank + 1) // world * align


def partial_layout(n_positions, hidden):
    """Byte offsets of one shard's partial (the layout dg_partial_bytes sizes): per position a float4
    {m, l, u, best}, an int32 argmax, a float sampled key and an int32 sampled index, then the
    self-conditioning numerator [N, d] float32; every field starts on a 256-byte boundary."""
    off, out = 0, {}
    for name, nbytes in (("stats", 16 * n_positions), ("idx", 4 * n_positions), ("skey", 4 * n_positions),
                         ("sidx", 4 * n_positions), ("o", 4 * n_positions * hidden)):
        out[name] = off
        off = (off + nbytes + 255) // 256 * 256
    out["total"] = off
    return out


def exchange_partials(partial, gathered, group=None):
    """All-gather one shard partial (flat uint8 tensor) into `gathered` ([world * nbytes]) in rank order."""
    world = tdist.get_world_size(group)
    if gathered.numel() != world * partial.numel():
        raise ValueError("gathered must hold one partial per rank")
    if tdist.get_backend(group) == "nccl":
        tdist.all_gather_into_tensor(gathered, partial, group=group)
    else:
        tdist.all_gather(list(gathered.view(world, -1).unbind(0)), partial, group=group)
    return gathered


class SplitStep:
    """One rank's part of a vocabulary-parallel step.

    p describes the whole head (p.vocab = the full vocabulary); W_shard / E_shard are
    this rank's rows [v0, v1) on its device.  Call with the step, the hidden states,
    the seeds and a StepBuffers; the outputs land in the buffers as with dg_denoise_step.
    """

    def __init__(self, p, W_shard, E_shard, v0, v1, group=None):
        self.p, self.W, self.E, self.v0, self.v1, self.group = p, W_shard, E_shard, v0, v1, group
        self.world = tdist.get_world_size(group) if tdist.is_initialized() else 1
        dev = W_shard.device
        self.ws = Workspace(p, dev)
        n = dg_partial_bytes(p)
        self.partial = torch.empty(n, dtype=torch.uint8, device=dev)
        self.gathered = torch.empty(self.world * n, dtype=torch.uint8, device=dev)

    def init(self, seeds, tokens, stream=None):
        """Canvas initialisation and reset of this rank's sampler state (identical on every rank)."""
        dg_canvas_init(self.p, seeds, tokens, self.ws, stream)

    def __call__(self, step, h, seeds, bufs, stream=None, selfcond=None):
        """One step; the self-conditioning vectors go to `selfcond` when given, else bufs.selfcond."""
        dg_denoise_partial(self.p, step, self.v0, self.v1 - self.v0, h, self.W, self.E, seeds, self.partial, self.ws,
                           stream)
        if self.world > 1:
            exchange_partials(self.partial, self.gathered, self.group)
            parts = self.gathered
        else:
            parts = self.partial
        dg_denoise_merge(self.p, step, self.world, parts, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                         bufs.lse, bufs.selfcond if selfcond is None else selfcond, self.ws, stream)
