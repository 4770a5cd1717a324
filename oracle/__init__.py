"""Plain float64 CPU oracle for the NVFP4 weight-streaming skinny GEMM and greedy verify.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or execute
anything in this package. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

The oracle shares no code with the CUDA library: no kernels, headers, tables or
constant generators. It is written from the definitions of the formats and of the
method, step by step, with no blocking or fusion:

* ``nvfp4``  -- E2M1 / E4M3 value sets, round-to-nearest-even with saturation, the
  two-level NVFP4 quantiser (per-tensor FP32 scale, per-16-element E4M3 block
  scale, E2M1 codes), dequantisation and the byte packing layout.
* ``gemm``   -- ``Y = X . dequant(W)^T`` in float64 with bf16 X.
* ``verify`` -- per-row argmax (lowest index on ties), the near-tie gap, the greedy
  accept length and the committed tokens.

Sources (web pages, cited by title and section):

* "Qwen3.8 on DGX Spark (GB10)" (hasso5703/dgx-spark-qwen38), section "The seven
  targets, and switching between them": the weights are NVFP4 with group size 16.
  The same page's introduction gives the vocabulary (248,320 rows) and the
  65,536-row slice.
* "TandemLLM" (0xBakeer/TandemLLM), introduction: the target checks every drafted
  token; at the first wrong guess it emits its own token. The same paragraph gives
  the one-ulp near-tie exception.
* "TandemLLM", "How it works" flowchart: keep the longest path the model agrees with.

The pages do not define the bit encodings. Where they are silent, this package takes
the plain readings listed in each function's docstring.

Every function is pinned by ``tests/test_oracle_*.py``. Nothing here is "parity
unpinned".
"""

from . import nvfp4, gemm, verify  # noqa: F401
