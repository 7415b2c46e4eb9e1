"""CPU oracle for the streamed NF4-LoRA training path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it.  It shares no code, table or constant generator
with the CUDA library; both sides take their inputs from ``synthetic``.

Everything here is plain and slow on purpose: numpy / PyTorch CPU in fp64
(exact fp32 where the method fixes fp32 arithmetic, e.g. the quantiser's
division and the dequantiser's multiply), no blocking, fusion or reordering
beyond what the definitions state.

Sources.  The pages ("Soup" README snapshot; soup-cli 0.72.0 -> 0.72.2 diff,
CHANGELOG [0.72.2] and docs/performance-and-quantization.md "Layer Streaming")
say only that the frozen base is quantised to NF4 once, ahead of training, and
that a streamed run feeds identical quantised bytes to identical kernels as a
resident run, and that the trainer is
a LoRA SFT trainer with gradient checkpointing.  They fix neither the codebook,
the block size, the absmax type, the nibble order nor the LoRA maths; where
they are silent the reading taken is stated in the function that takes it.

Pins (tests/test_oracle_*.py): closed-form codebook invariants and an
independent inverse-normal routine; brute-force argmin on every element;
the round trip deq o quant o deq == deq; B = 0 reduces LoRA to the base linear;
central finite differences for every analytic gradient; S = 1 attention equals
the V projection; RoPE at position 0 is the identity; the SmolLM2-135M
parameter count the pages print; the loss at init near ln(V); for the
double-quantised absmax, the E4M3 table and rounding against torch's
float8_e4m3fn, exact round trips on representable blocks and the half-ulp
error bound.
"""
