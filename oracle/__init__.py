"""CPU oracle for the compressed-KV hot path — TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 restatement of what the method computes, written from the
pages that describe it (TurboESM, gist.science "TurboESM: Ultra-Efficient 3-Bit
KV Cache Quantization for Protein Language Models ..."; TurboQuant,
7minutos.es "KV cache está consumiendo tu VRAM ... TurboQuant", sudonull.com
"TurboQuant: compresión 6x de LLM KV-cache", news.hada.io TurboQuant summary).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package. It shares no code with the CUDA library
(``kv_cache_vector_rope_b200``) and never imports it; the only common inputs
come from the seeded generators in ``synth``.

Modules:
  codebook   Lloyd-Max on the post-rotation coordinate law; empirical Lloyd.
  quantize   RoPE, rotation, norm, bucketize, pack, QJL signs.
  attention  scores over packed planes, softmax attention, dequantisation.
  calib      per-head SVD basis composed with the random rotation.
  search     estimated-score and exact top-k over a compressed corpus.

Every function is pinned by tests under ``tests/test_oracle_*.py`` against
closed forms, printed worked examples, brute force or statistical identities.
"""
