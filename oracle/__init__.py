"""CPU oracle of the denoising step: plain, slow, float64 (float32 where the
float32 key is the definition).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import or run this package.
The product path (the CUDA library and its Python binding) never imports it
and has no CPU fallback.  It shares no code with the CUDA path: the only
module both use is ``synth`` (seeded input generators, no method arithmetic).

Modules:
  philox  -- Philox4x32-10 from the SC'11 paper.
  flog    -- the float32 log / Gumbel transform the keys are specified with.
  step    -- the step: temperature, logits, entropy, argmax, Gumbel-max draw,
             entropy-bounded selection, renoise, stop.
  replay  -- the sampler replayed on given float32 logits.
  loop    -- the adaptive loop with final commit.
  blocks  -- block-by-block generation (encode & append) over the loop.
  selfcond -- the self-conditioning signal read as the expected embedding
             (its CUDA side is not built yet).

Parity pins: every function is checked in ``tests/test_oracle_*.py`` against
something other than itself (closed forms, brute force in exact arithmetic,
independent library routines, invariants, chi-square).  The composed step has
no worked example on the pages: its end-to-end values are pinned only through
its parts.
"""
from . import blocks, flog, loop, philox, replay, selfcond, step
from .blocks import generate_blocks
from .loop import denoise_loop
from .replay import replay_step
from .step import Params, denoise_step

__all__ = ["blocks", "flog", "loop", "philox", "replay", "selfcond", "step", "Params",
           "denoise_step", "denoise_loop", "generate_blocks", "replay_step"]
