"""Float64 CPU oracle for the quantized KV cache -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct restatement of what the
quantized-KV decode path computes.  It is the checker for the CUDA library, not
part of it: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never imports, links or calls anything here, and nothing here
imports the CUDA library; the two share only the seeded input generator
(``quantized_kv_cache_18_b200.workloads``), which holds none of the method's
arithmetic and which this package does not import either (inputs arrive as
arrays).

Sources (web pages on KV-cache quantization; cited by title and section):

* [P1] "KV-cache compresse et modeles 4-bit : la compression s'impose comme le
  premier levier d'inference" (ai-automate.fr) -- section "Minima-KV : la
  compression sans eviction" (partial attention states merged by a globally
  normalised online softmax).
* [P2] zubnet.ai survey "KV cache compression techniques: H2O, KIVI, MLA,
  StreamingLLM" -- paragraph "Famille deux, c'est la quantification" (KIVI keys
  per channel / values per token; TurboQuant rotation + 1-bit QJL).
* [P3] "La compression du cache KV est une decision d'infrastructure, pas un
  debat sur les modeles" (encorp.ai) -- sections "... quand la HBM, pas les
  FLOPs, est votre plafond" (70B bytes per token) and "TurboQuant est le choix
  de portabilite, pas le gagnant universel" (random rotation, precomputed
  scalar quantizer, QJL on the residual).
* [P4] "Quantification du KV-Cache : TurboQuant et l'etat de l'art en 2026"
  (patricehuetz.fr) -- sections "Le probleme : le KV-cache, gouffre silencieux"
  (memory formula), "KIVI (2024)", and "TurboQuant : les cinq innovations"
  items 1 (rotation), 2 (Lloyd-Max), 3 (bit packing), 4 (residual window).

Where the pages leave a step open the oracle takes the plainest reading and
says so in the function that implements it.  Every function below is pinned
by a ``-m "not gpu"`` test against something other than itself (closed forms,
the pages' worked numbers, exact rational arithmetic, brute force, textbook
tables) except where its docstring says "parity unpinned".
"""
