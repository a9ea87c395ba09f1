"""CPU oracle for the TTT-KV fast-weight layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct float64 numpy.  It is the yardstick the CUDA
path is measured against and is never part of that path: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  It shares no code with the CUDA library (no kernels, headers,
helpers or table generators); the only thing both sides consume in common is
the seeded input module ``ttt_synth``.

Contents
  ttt_linear  -- linear fast weight trained on the negative inner-product
                 binding loss (token-by-token recurrence) and the equivalent
                 causal linear-attention sum; the backward pass (gradients of
                 a linear functional of the outputs and final state).
  lact        -- large-chunk TTT with a SwiGLU fast-weight memory: chunk
                 gradients, GD / momentum / Muon (Newton-Schulz) updates, row
                 L2 normalisation, causal and bidirectional ordering.
  lact_backward -- gradients of the LaCT layer through its chunk loop
                 (float64 torch restatement of the forward, differentiated by
                 torch.autograd; pinned to the numpy oracle and to central
                 differences).
  window_attention -- causal sliding-window softmax attention, and the LaCT
                 language layer (memory + window attention, outputs summed).

Every function names the passage of the pages it follows.  Pins (checks
against facts that are not this code) live in ``tests/test_oracle_*.py``.
"""
from .ttt_linear import (ttt_linear_recurrent, ttt_linear_attention_sum,  # noqa: F401
                         ttt_linear_backward)
from .lact import (lact_forward, lact_read, lact_chunk_gradients, newton_schulz,  # noqa: F401
                   silu, silu_prime, LaCTState)
from .window_attention import sliding_window_attention, lact_layer_forward  # noqa: F401
