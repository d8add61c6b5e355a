"""CPU oracle for low-bit KV-cache quantize-append and decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links this package:
only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline / reference leg may use
it.  It shares no code, table or constant generator with the CUDA library; both sides take
their inputs from `quantized_decode_attention_append_b200.synth`, which holds no method
arithmetic.

Plain, slow, vectorised numpy.  Where a floating-point value decides an integer code, the
decision is taken exactly (fp64 comparisons whose operands are exact), on fp32 transform
outputs computed in the evaluation order the format fixes.  Attention and reconstruction
are fp64.

Sources (web pages; cited by title and section):
  * "Fourier Magnitude KV Cache Quantization" (forum thread): post 6 sections "Corrected
    semantics", "Minimal recipe", "Milestone", "Debunk audit", "The winning recipe"; the
    reply's sections "The three controls I would try first", "The finite-phase
    implementation and the physical codec may be worth separating", "Why
    attention-visible distortion seems especially useful here".
  * "E21W: known 3-bit KV cache methods on the 4B ... (proxy queries)": "What I tested",
    "Result".
  * "E22L: Can 4-bit keys and 2-bit values hit a 1M-token memory budget?": "What I tested",
    "Result".
  * llama.cpp issue #21385 "Per-head adaptive KV cache quantization": "Finding 1".

Parity status: every function here is pinned by `tests/test_oracle_*.py` except the NF4
level values themselves ("parity unpinned" beyond the properties of their construction; the
pages name NF4 but print no table).
"""
