"""fp64 CPU oracle of the Cosmos 3 Mixture-of-Transformers layer hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package's
smoke check and the CPU-baseline leg of the benchmark may import it.  The CUDA
library never calls into it and shares no code with it; the two meet only in
the seeded inputs of the ``synth`` package.

Everything here is plain numpy in float64: each bf16 input is promoted exactly
and no intermediate is rounded.  Library primitives (matmul, exp, sin, cos)
serve as single steps; there is no blocking, fusion or reordering beyond what
the definitions state.  Each function names the passage it follows:

  * "Cosmos 3 方法原理全解" (cnblogs): §2 packed sequence S=[S_AR, S_DM] and
    its internal order; §2.2 clean/noisy condition mask; §3 MoT: two weight
    sets, causal AR attention and full DM attention over [K_AR; K_DM]; §4.2
    domain action projections W_in / W_out; §5 unified 3D mRoPE, real-time
    step sizes and the 15000 offset; §6.3 the linear flow path, per-modality
    noise levels and the flow shift; §7.2-7.3 the Euler sampler step and
    classifier-free guidance; §12.4 the stacked model sizes.
  * "NVIDIA 发布 Cosmos 3 系列四个开放权重世界模型", "流式生成如何工作":
    time-causal block attention with a key/value cache.

Where the pages are silent the oracle takes a stated reading, given in the
docstring of the function concerned (norm type, RoPE base and pairing, t/h/w
split, EOS/BOG region, position formulas, streaming commit, the head of a
stack, the inference grid of the shift).  Every function is pinned by tests
under ``tests/test_oracle_pins.py`` (closed forms, invariants, brute force and
the values the pages print) except where a docstring says "parity unpinned";
none does.  No page prints a layer output, so a layer's numerical value is
pinned only through those tests.
"""

from . import layout, rope, mask, layer  # noqa: F401
