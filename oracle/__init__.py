"""CPU oracle for the int4 / FP8 mixture-of-experts FFN layer.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the layer computes, in numpy (fp64 wherever the pages do
not fix a precision).  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import it.  The CUDA library never
imports, links or calls anything here, and nothing here uses the CUDA library.

Sources (web pages; cited by title and section):
  [P1] "1 卡跑通 Llama 4：从本地部署到多模态推理的完整路径" (discosf.com),
       sections "混合专家路由" (MoE.forward: router scores, top-k, scatter_add_,
       shared expert) and "FP8 / Int4 混合量化" (int4_row_quantize).
  [P2] "Meta Llama Models Llama 4 单卡量化推理与选型指南" (lshu.cn),
       section "量化环节做了什么" (bmm_nt, FP8 row / int4 group-128 weights,
       zero points equal to zero) and the table "三条推理路径差异".
  [P4] "Llama" (illegalscreed.cn), introduction (16 experts; 128 routed + 1
       shared experts).
  [P5] "Llama 开源模型系列" (docs.ifdog.com), sections "MoE 架构详解" (router =
       linear layer + softmax, top-1 / top-8), "SwiGLU：门控激活的数学" and
       "RMSNorm：为什么去掉减均值也能工作".

Where the pages are silent or ambiguous the oracle takes a stated reading;
every function states the reading it uses.

Parity status: every function here is pinned by CPU tests against worked
examples, brute force, closed forms, library special cases or invariants
(tests/test_oracle_*.py).  No function is "parity unpinned".
"""
from . import quant, route, ffn, norm  # noqa: F401
