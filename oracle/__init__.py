"""CPU oracle for the Mel-Band RoFormer core forward (stft_repr -> per-bin complex masks).

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 NumPy restatement of
what the method computes, written from the pages' description of the model.  Only the
test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
it.  It shares no code with the CUDA path and imports nothing from it.

Modules:
  tables  - Slaney mel filter bank, its binarised band incidence, the gather/average tables
  model   - band split, axial transformers (RoPE, gated attention, GELU feed-forward),
            mask estimator with GLU, overlap average, parameter counting

Pins (tests/test_oracle_*.py): per-band bin counts and overlap counts printed by the
pages, parameter counts 228,202,788 and 217,301,852, MAC counts of the FLOP accounting,
RMSNorm / RoPE / softmax / attention invariants, brute-force attention on tiny inputs,
partition of unity of the overlap average, batch stacking.  The end-to-end masks on
random weights have no printed values: beyond the component pins their parity is
unpinned, and the CUDA path is pinned to this oracle only.
"""
from . import tables, model  # noqa: F401
