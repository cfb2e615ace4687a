"""CPU oracle of the SoulX-FlashHead Lite flow-prediction transformer.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously-correct CPU
restatement of what the hot path computes, used to check the CUDA library. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it. The product path (``audio_driven_talking_b200``) never does, and the
two share no code: the only common module is ``synth_inputs`` (the seeded input
generator, which holds none of the method's arithmetic).

Modules:
  model  - vectorised numpy oracle: timestep conditioning, RoPE, block, flow
           prediction, 4-step sampler (float64, float32, or float32 with the
           bf16 operand rounding the bf16 configurations state).
  brute  - float64 per-token loop recomputation of one block (small sizes),
           written independently of ``model`` to pin it.

Parity status of each function is listed in ``model``'s module docstring.
"""
from .model import (Config, CFG0, CFG1, CFG2, CFG3, CFG4, Weights, make_weights,
                    time_conditioning, rope_angles, block_forward, predict_flow,
                    sample_slice, param_count)

__all__ = ["Config", "CFG0", "CFG1", "CFG2", "CFG3", "CFG4", "Weights", "make_weights",
           "time_conditioning", "rope_angles", "block_forward", "predict_flow",
           "sample_slice", "param_count"]
