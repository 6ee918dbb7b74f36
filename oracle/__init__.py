"""IsoQuant oracle: a plain, slow, fp64 CPU restatement of the packed-3-bit KV path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product (the C-ABI library, its kernels
or the Python binding) imports, links or executes anything in this package.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl
reference`` legs of ``bench.py`` may call it.  It shares no code, table or
constant generator with ``rotated_bit_kv_iq_b200``; the two meet only through the
seeded input generator module, which holds none of the method's arithmetic.

Sources (web pages; cited by title and section):
  [RQ-news]  "RotaryQuant" write-up, rebasdaily.com topic page of 2026-08-14
             (sections "妙处不只是压缩，而是不再展开", "省内存，不等于更快").
  [RQ-abs]   RotaryQuant, arXiv 2608.08081, arxivdaily entry, English abstract.
  [TQ-RQ]    "压缩与速度的博弈——TurboQuant 和 RotorQuant 的真相", zhichai.net
             (sections "为什么压缩 KV 缓存这么难？", "Beta 分布的魔力",
             "Lloyd-Max 最优量化", "真正的瓶颈", "三种变体").
  [RQ-wiki]  "RotorQuant：LLM KV 缓存压缩的“几何革命”", sd114.wiki
             (section "3. V 缓存的逆旋转修复").

Modules:
  codebook   Lloyd–Max scalar quantiser for N(0,1) and N(0,1/d)    -- pinned
  rotation   Sylvester WHT, quaternion SO(4) blocks, seed -> params -- WHT/SO(4)
             pinned; the seed -> parameter mapping is "parity unpinned" (the
             pages publish no parameter values; only the C library's host
             generator is checked against it, bit for bit)
  encode     norm -> WHT -> SO(4) -> threshold search              -- pinned
  packing    the 48-byte code layout (ours; the pages fix none)     -- pinned by
             its written specification and hand-made fixtures only
  attention  decode attention on the packed cache, two ways        -- pinned
  opcount    instrumented op counter for the rotation              -- pinned
"""

from . import codebook, rotation, encode, packing, attention, opcount  # noqa: F401
