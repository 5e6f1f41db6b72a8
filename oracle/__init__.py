"""CPU oracle for the Z-Image S3-DiT forward and its FlowMatch-Euler step.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, step-by-step CPU
statement of what the GPU library computes, used to check it.  Only the test
suite, the smoke check and the benchmark's CPU-baseline leg may import it; the
product path (the CUDA library and its Python binding) never does, and fails
loudly instead of falling back to it.

It shares no code with the CUDA path.  Its only shared dependency is the seeded
input generator ``zimage_inputs`` (shapes and random numbers, no arithmetic).

Floating point is fp64 (NumPy) unless a caller asks for another dtype; weights
are the bf16-rounded values both sides receive, upcast.

Modules:
  zimage_ref    -- the transformer forward, step by step
  scheduler_ref -- shifted sigma schedule, Euler update, CFG combine, denoise loop
  brute         -- scalar-loop fp64 restatements used to pin the above on tiny inputs

Parity unpinned: the absolute values of a full-stack output.  The pages print
no worked example of the transformer's output, and trained weights are not
available, so full-stack values are pinned only through the component pins,
invariants and exact counts in tests/test_oracle_*.py.
"""
