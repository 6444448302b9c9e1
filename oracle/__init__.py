"""Plain fp64 CPU oracle for the same-step KV chunk-attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports, links or
runs this code; only the tests, the smoke check and the bench's CPU-baseline
leg do.  It shares no code with the CUDA path: the two meet only through the
seeded input generator, which holds no arithmetic of the method.

The oracle computes what the pages define, written out plainly:

* ``schedule``  - the chunk / ring bookkeeping of the PhysisServe Wan2.2-5B
  model card ("Inference profile" table and the paragraph under it), kept as
  an explicit list of ring slots with eviction of the oldest chunk;
* ``rope``      - 3D (frame, height, width) rotary embedding, blog "Learning
  Video Generation from the Wan2.2 Source Code", chapter 4, section "3D RoPE";
* ``attention`` - softmax attention over a key set, by its definition, plus a
  brute-force masked dense version used to pin it (blog chapter 8 for the
  FLOP count);
* ``euler``     - the flow-matching Euler update, blog chapter 5 ("UniPC")
  and chapter 1 ("From DDPM to Flow Matching");
* ``session``   - one stream's same-step KV history driven through a whole
  chunk schedule (model card, "Inference profile");
* ``projection`` - the q, k, v linear layers and the QK-Norm (RMSNorm of q
  and k), blog chapter 4, end of "3D RoPE: Letting Tokens Know Where They
  Are".

Every function is pinned by tests under tests/ that do not re-type its
formula: closed forms, invariants, brute force and the pages' printed numbers.
"""
