"""Plain, slow, fp64 CPU oracle for the TurboQuant KV-cache hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call,
link or execute anything under ``oracle/``.  The only permitted users are
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py``.  The oracle shares no code,
tables or constant generators with the CUDA library: it is a second,
independent statement of the method, written for a reader to check by eye
against the pages it cites.

Pages cited, by title (sections are given per function):

  [inferrs] "inferrs & TurboQuant：本地 LLM 推理的内存革命"
  [tqai]    "TurboQuant：让大模型本地推理内存占用降低80%的KV缓存压缩技术"
  [fwht]    "TurboQuant：用Rust核心与FWHT预处理实现LLM推理的4-bit KV缓存量化"
  [google]  "Google 最新極限壓縮算法，砸碎大模型本地部署的內存墻，8 倍提升！"

Arithmetic is fp64 throughout, except where floating point decides an
integer that the pages do not fix and the kernels decide in fp32 (the int8
boundary-layer scale and rounding, see ``quantize.encode_int8``); there the
oracle performs the same IEEE fp32 operations so that both sides take the
same decision.

Modules
-------
rng        SplitMix64 stream, rotation signs, Gaussian QJL sketch matrix.
rotation   Sylvester Hadamard matrix, random-sign rotation and its inverse.
codebook   Lloyd-Max codebook for the rotated-coordinate density, and the
           Gaussian Lloyd-Max solver used only to pin it.
quantize   norm, codes, bit packing, QJL residual bits, int8 mode,
           dequantisation.
attention  decode attention over dequantised vectors, Sparse-V bounds.
paging     the paged cache layout: which block row holds a token.
"""

from . import rng, rotation, codebook, quantize, attention, paging  # noqa: F401
