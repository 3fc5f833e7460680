"""Plain fp64 CPU oracle of the MoGA visual-attention layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this package: only the tests, the package's smoke check and the CPU
baseline leg of the benchmark script use it.  It shares no code with the CUDA
library; the only module both sides use is `synth`, the seeded input
generator, which holds none of the layer's arithmetic.

Every function reads its inputs exactly into float64 and computes the plain
definition from the pages, step by step, with numpy's matmul/exp/argmax as
library primitives.  No tiling, fusion or reordering beyond the definition:
where a computation is split (rows of an attention output computed in chunks),
the pieces are independent by definition.

Citations name the page and its section:
  * papernotes.org ICLR 2026 note "MoGA: Mixture-of-Groups Attention for
    End-to-End Long Video Generation" -- "note", with its sections 关键设计
    (key designs) 1-4 and 训练设置 (training setup);
  * the jxzklqfsx.com Chinese translation of the paper -- "translation",
    section 方法 (method) with 混合分组注意力 (MoGA), 组平衡损失 (group
    balancing loss) and 时空分组注意力 (STGA);
  * the xugj520.cn blog "把 1 分钟 480p 视频塞进 58 万 token" -- "blog", with its
    numbered sections (2.3 router sketch, 3.2 shot-aligned local windows,
    9 failure table).

Parity status per function (what pins it) is listed in each module header.
"""
from . import route, permute, stga, attention, layer  # noqa: F401
