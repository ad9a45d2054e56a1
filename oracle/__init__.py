"""Float64 CPU oracle for the canvas denoise-sampling stage.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call, link
or execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` use it.  It shares no code with the
CUDA library (``discrete_diffusion_decoding_b200``) and imports nothing from it.

Each function restates, in plain and deliberately unoptimised NumPy float64,
what the pages on DiffusionGemma say one denoising step computes:

* uniform-state noise: a noised position holds a token drawn uniformly from the
  vocabulary ("Uniform State Diffusion" sections of the marrrang.tistory.com
  deep dive and of the juhoplayground overview);
* per-position token distributions over the whole canvas, their entropy and the
  arg-max prediction (deep dive, "reverse diffusion" steps 3-5);
* the entropy-bounded sampler: keep confident tokens, re-noise the others with
  random vocabulary tokens (juhoplayground "inference mechanism"; deep dive
  sampling-settings table: entropy bound 0.1);
* self-conditioning: the probability-weighted token embedding softmax(z/T)·E
  (juhoplayground "inference mechanism");
* the temperature schedule, linear 0.8 -> 0.4 over at most 48 steps, and the
  two-fold adaptive stop: mean canvas entropy below 0.005 AND the predictions
  unchanged over two consecutive steps (deep dive "Two-Fold Adaptive Stopping").

Parity status per function is listed in each module header.
"""

from . import philox, stage, decode  # noqa: F401
