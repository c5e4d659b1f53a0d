"""Plain CPU oracle for the Block-GTQ packed-cache decode path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call, link
or execute anything in this package: only ``tests/``, ``__graft_entry__.smoke``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

Everything here is written for a reader to check by eye against the method
as stated on the pages of "RoPE-Aware Bit Allocation for KV-Cache
Quantization" (Liang, Zhang, Jia; chatpaper summary / arXiv 2606.24033
abstract, the blockgtq README) and the TurboQuant-MSE encoder those pages
build on.  Arithmetic is float64 (or exact Python integers) unless a step is
defined to round (the fp32 tables, the fp16 norms).  Library primitives used
as steps: ``numpy.linalg.qr``, ``numpy`` matmul / sort / searchsorted.  There
is no blocking, fusion or reordering beyond the plain definition.

Modules
-------
lloyd_max   Gaussian Lloyd-Max scalar quantiser tables (TQ-MSE's codebook).
haar        SplitMix64 -> Box-Muller -> Householder-QR Haar rotations.
energy      label-free per-RoPE-block Q/K energy score (exact integers).
allocate    greedy integer bit allocation by marginal gain; group layout.
tqmse       rotate / normalise / quantise one row; bit-pack a record.
attention   dense decode attention from packed records.
model       the per-(layer, KV head) tables and the cache-level calls.
diag        the per-layer logit MAE of a packed key cache (K only).
rope        rotary position embedding of key rows (the fused RoPE + encode).
"""
