"""The vocabulary split's exchange over NCCL on the GPU, in a one-rank process group.

Two ranks on one GPU would be kernels waiting on one another on a single device, which
this test never runs; a one-rank NCCL group still drives the product's exchange code
(`vocab_parallel.exchange_partials`, an NCCL all-gather of device buffers) and the
SplitStep class end to end on CUDA tensors.  The gathered partial must equal the
rank's own, and the merged step must equal the single-call step (identical argmax,
accept flags and tokens; entropies and vectors to rounding), as in the one-GPU shard
tests.  Runs in a spawned child so that the test process's CUDA context and the
process group stay apart.
"""

import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(port, q):
    import sys
    from datetime import timedelta
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1", LOCAL_RANK="0",
                      NCCL_NVLS_ENABLE="0")
    try:
        import torch
        import torch.distributed as dist

        import synth
        import discrete_diffusion_decoding_b200 as dg
        from discrete_diffusion_decoding_b200 import vocab_parallel as vp

        torch.cuda.set_device(0)
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60))
        try:
            V, d, C = 8192, 512, 2
            W = synth.weights(V, d, seed=51).cuda()
            h = synth.gaussian_hidden(256 * C, d, seed=52).cuda()
            seeds = torch.tensor([5, 6], dtype=torch.int64, device="cuda")
            p = dg.params(C, V, d)
            # the single call
            ws, ref = dg.Workspace(p), dg.StepBuffers(p)
            dg.dg_canvas_init(p, seeds, ref.tokens, ws)
            ref.h.copy_(h)
            dg.dg_denoise_step(p, 1, ref.h, W, W, seeds, ref.tokens, ref.entropy, ref.argmax, ref.accept, ref.lse,
                               ref.selfcond, ws)
            # the split path: the shard partial, the NCCL all-gather, the merge
            st = vp.SplitStep(p, W, W, 0, V)
            bufs = dg.StepBuffers(p)
            st.init(seeds, bufs.tokens)
            bufs.h.copy_(h)
            dg.dg_denoise_partial(p, 1, 0, V, bufs.h, W, W, seeds, st.partial, st.ws)
            gathered = torch.zeros_like(st.partial)
            vp.exchange_partials(st.partial, gathered)
            torch.cuda.synchronize()
            same_bytes = bool(torch.equal(gathered, st.partial))
            dg.dg_denoise_merge(p, 1, 1, gathered, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                                bufs.lse, bufs.selfcond, st.ws)
            flags, _, _ = dg.dg_stop_check(p, st.ws)
            # and SplitStep.__call__ itself, on a fresh canvas
            bufs2 = dg.StepBuffers(p)
            st.init(seeds, bufs2.tokens)
            bufs2.h.copy_(h)
            st(1, bufs2.h, seeds, bufs2)
            torch.cuda.synchronize()
            out = {"backend": dist.get_backend(), "same_bytes": same_bytes, "flags": list(flags)}
            for name, b in (("ref", ref), ("merged", bufs), ("call", bufs2)):
                out[name] = {k: getattr(b, k).cpu().numpy() for k in
                             ("entropy", "argmax", "accept", "tokens", "lse", "selfcond")}
            q.put(("ok", out))
        finally:
            dist.destroy_process_group()
    except Exception as e:  # reported to the parent
        import traceback
        q.put(("error", traceback.format_exc() + repr(e)))


def test_nccl_exchange_and_merge_one_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    proc = ctx.Process(target=_child, args=(_free_port(), q))
    proc.start()
    try:
        status, out = q.get(timeout=300)
    finally:
        proc.join(timeout=60)
        if proc.is_alive():
            proc.kill()
    assert status == "ok", out
    assert out["backend"] == "nccl"
    assert out["same_bytes"], "a one-rank all-gather must return the rank's partial unchanged"
    ref = out["ref"]
    far = np.abs(ref["entropy"] - 0.1) >= 1e-3          # accept decisions away from the bound
    for name in ("merged", "call"):
        got = out[name]
        assert np.array_equal(got["argmax"], ref["argmax"]), name
        assert np.array_equal(got["accept"][far], ref["accept"][far]), name
        assert np.array_equal(got["tokens"][far], ref["tokens"][far]), name
        assert np.abs(got["entropy"] - ref["entropy"]).max() <= 1e-4, name
        assert np.abs(got["lse"] - ref["lse"]).max() <= 1e-4, name
        rel = np.linalg.norm(got["selfcond"] - ref["selfcond"], axis=1) / np.linalg.norm(ref["selfcond"], axis=1)
        assert rel.max() <= 2e-2, name
