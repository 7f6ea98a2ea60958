"""fp64 CPU oracle for absorbed MLA decode with decoupled RoPE.

TEST INFRASTRUCTURE ONLY.  This package is the checker, not the product: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may import it.  The CUDA library under ``mla_latent_kv_45_b200``
never imports, links or calls anything here, and nothing here imports the
CUDA path; the two share no arithmetic.  The only module both sides use is
``mla_latent_kv_45_b200.synth``, which draws seeded random inputs and holds
none of the method's arithmetic.

Sources (the five web pages on the subject, cited by title and section):

* "解耦 RoPE（MLA 下）" (Decoupled RoPE, MLA part 2; agent.namiai.tech) --
  the hand-worked 3-token example (§四), the per-token inference flow (§五),
  the 576 arithmetic (§六) and a PyTorch ``MLA`` with ``rope`` /
  ``forward_naive`` / ``forward_absorbed`` (§七).
* "从零理解 MLA" (momoyeyu.github.io, llm-mla) -- the compression, absorption,
  query-compression and decoupled-RoPE equations (sections 低秩联合压缩,
  矩阵吸收, 查询压缩, 解耦 RoPE), ``absorbed_step`` with a ``[c ; k_R]`` cache
  row, and the DeepSeek-V2 dimensions (实际配置).
* "Hands-on DeepSeek MLA" (ackingliu.top repost) -- the RMSNorm class.
* "构建DeepSeek-V3：多头潜在注意力(MLA)架构" (juejin.cn) -- c_KV = RMSNorm(W_dkv x).
* "旋转约束下的压缩：从 RoPE 到 DeepSeek MLA" (xuquant.com) -- context only.

Parity status per function is listed in ``oracle.mla_oracle.__doc__``.
"""

from .mla_oracle import *  # noqa: F401,F403
