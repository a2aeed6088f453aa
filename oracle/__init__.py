"""CPU oracle for the batch-1 persistent decode step.

TEST INFRASTRUCTURE ONLY.  Only the tests, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import or run
anything in this package.  The product path (the CUDA library and its Python
binding) never calls it, and shares no code, headers or tables with it; the only
common dependency is the `synth` package of seeded input generators.

What it computes: one decode step of a dense GQA decoder or of an MLA + MoE
decoder at batch 1, in float64, with the activation rounding points of the
model definition (bf16 for the bf16/fp8 workloads, fp32 for the fp32 one).  The
pages describe the model family (TileRT 是什么, §五 5.2 模型结构支持: MLA, MoE with
256 routed experts and 8 active, dense first layers) and the KV buffers
(§五 5.3 内存管理: kv_cache and pe_cache) but print no formula; every formula
here is the plain textbook reading, each one named where it is implemented.

Pins (tests/test_oracle_*.py, all `-m "not gpu"`): float64 brute force for
GEMV and softmax, the E4M3 code table against the format definition and
torch.float8_e4m3fn, bf16 rounding against torch, RoPE norm preservation and
relative-position invariance, incremental decode == full causal recompute,
context length 1 returns V, one expert with top-1 == the dense MLP, router
weights sum to 1, absorbed MLA == unabsorbed MLA, split-KV log-sum-exp combine
== one softmax, argmax == numpy first-max; and closed forms of special cases that bypass
the step code (test_oracle_structure.py): zeroed output projections pass the embedding
through, a one-layer FFN-only step, two-position attention as a sigmoid mix (dense and MLA),
two-expert router weights as a sigmoid pair.  Parity of whole-model values beyond
these pins is unpinned: the pages print no worked example.
"""
