"""CPU oracle for the DeepSeekMoE FP8 layer forward pass.

TEST INFRASTRUCTURE ONLY. This package is the slow, plain reference that the
CUDA path is checked against. Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it. The product library never
calls it, and it shares no code with the CUDA sources: it is written from the
method's equations, in float64 numpy, step by step.

Sources (web pages about the DeepSeek-V3 technical report, arXiv 2412.19437):

* "DeepSeek-V3 Teknik Raporu" (xyznot.com/tr/paper/2412.19437), section
  "Yöntem", part 2 "Yardımcı Kayıpsız Dengelemeli DeepSeekMoE": the FFN output
  equation for h'_t, the sigmoid affinity s_{i,t}, the biased Top-k gate
  g'_{i,t}, the normalised gate g_{i,t} and the bias update with gamma=0.001.
  Section "Temel fikirler", bullet "FP8 Karma Duyarlıklı Eğitim": E4M3 on all
  tensors, 1x128 activation tiles, 128x128 weight blocks, FP32 promotion of
  the accumulation every N_c = 128.
* "DeepSeek-V3 Technical Report" (xyznot.com/fr/paper/2412.19437), the French
  copy of the same guide: "Méthode" part 2 and "Idées clés", same content.
* "[논문 리뷰] DeepSeek-V3 Technical Report" (nubint.ai), "제안 방법": FP8
  mixed precision with tile-wise and block-wise quantisation.

Modules:
  e4m3  - the E4M3 format (decode table, round-to-nearest-even encoder) and
          bf16 / fp32 rounding helpers.
  moe   - every step of the layer: quantisers, router, top-K, gates,
          permutation, expert FFN, combine, bias update, and the full forward.

Parity status: every function is pinned by tests in tests/test_oracle_*.py
against closed forms, brute force, library routines (torch's float8 / bf16
casts) or invariants. No function is "parity unpinned"; the end-to-end values
of the five workloads have no worked example on the pages and are pinned only
through those per-step pins and the special-case reductions (see the tests).
"""
from . import e4m3, moe  # noqa: F401
