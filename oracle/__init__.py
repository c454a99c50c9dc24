"""CPU oracle for exact tiled attention: TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct statement of what the GPU
path computes.  It is used by ``tests/``, by ``__graft_entry__.smoke()`` and by
``bench.py``'s CPU-baseline leg, and by nothing else: the product path (the
C-ABI library and its Python binding) never imports it and has no CPU
fallback.  It shares no code, tables or helpers with the CUDA sources.

Modules
-------
attention  fp64 attention by its definition (full masked score matrix per
           document and head), the online-softmax recurrence replayed step by
           step, and a per-row evaluator for sampled checks at full size.
attention_bwd
           fp64 gradients (dQ, dK, dV) of the same definition, for the
           backward pass that follows the forward.
mxfp8      bit-exact E4M3 / E8M0 block quantiser and exact dequantiser.
schedule   the heaviest-first work list the schedule-build step must emit.

Sources (titles of the pages the method is taken from):
  * "FlashAttention và IO" (aihero.vn), sections "Ma trận trung gian là một
    khoản chi phí" and "Softmax qua nhiều khối cần thống kê chạy".
  * "FLAMIA: Blackwell Üzerinde Hızlı ve Nedensel Olarak Güvenli Eğitim İçin
    Flash Mikro-Ölçeklemeli Dikkat Mekanizması" (blog.edumints.com), section
    "FLAMIA Mimarisi ve Temel Tasarım İlkeleri".
  * "FlashAttention, pelatihan multi-GPU, dan kuantisasi bobot"
    (indonesian.itimpress.au), section 1.

Every function in this package has at least one pin in
``tests/test_oracle_*.py`` that checks it against something other than
itself (the pages' worked example, closed forms, a library routine on a
special case, or 50-digit brute force).
"""
