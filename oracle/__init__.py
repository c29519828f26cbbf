"""CPU oracle of the DeepSeekMoE layer forward with FP8 block scaling.

TEST INFRASTRUCTURE ONLY: tests/, the smoke check and the benchmark's CPU
baseline may import this package; the CUDA library and its Python binding
never do.  It shares no code with them; the only common dependency is the
seeded input generator in ``synthetic``.

Every function follows "DeepSeek-V3 Technical Report" (notes page), sections
"DeepSeekMoE and auxiliary-loss-free load balancing" (sigmoid affinity,
bias for selection only, normalised gates, batch-wise load monitoring and the
gamma update, node-limited routing) and "FP8 mixed precision training"
(1x128 activation tiles, 128x128 weight blocks, E4M3, online amax scaling,
FP32 accumulation), in FP64 where the method leaves the precision open.  The
readings that fix what the pages leave open are listed in moe_oracle.c.

Parity status: every function here is pinned by tests that do not re-run the
oracle's own formula (exact rational arithmetic, high-precision decimals,
library routines on special cases, brute-force enumeration, hand-written
golden values).
"""
from .oracle import *  # noqa: F401,F403
