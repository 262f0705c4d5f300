"""fp64 CPU oracle for the flow-map block draft and its prefix verify.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library; the two meet
only in the seeded input generators of ``fm_synth``.

Sources (web pages about FlashMap; cited by title and section):

* P1  "FlashMap并行草拟加速大模型解码" (zh)
* P2  "Polymathic AI и исследователи из Princeton выпустили FlashMap — модель-черновик
      Flow Map для декодирования LLM в 6,14 раза быстрее" (ru)
* P3  eskul.ir "FlashMap 16-token drafter, 6x faster Qwen3" (fa)
* P4  the-ai.news "Polymathic AI / Princeton FlashMap, acceleratore di decoding LLM" (it)
* P5  "FlashMap Drafts 16 Dependent Tokens at Once, Hitting 6.1x Faster Decoding" (en)

Modules:

* ``flashmap``  vectorised fp64 draft (context projection, conditioning,
  DiT blocks, LM head, token selection) and verify (greedy, stochastic,
  tree).  Used at every size.
* ``loops``     the same draft written with plain Python loops, for tiny
  shapes only; an independent second formulation.
* ``toy_flow``  the exact flow of a two-mode data distribution ("new york" /
  "san diego"), used to check the flow-map update and shared-noise drafting.

Parity status: the verify functions are pinned by exact enumeration of the
target distribution (at temperatures 1, 2 and 0.5) and by the
greedy-equals-target-greedy invariant; the zero-DiT draft by hand-computed
fixtures, one single-step and one two-step (the chain between flow-map
steps at a sampling temperature other than 1); attention, LayerNorm, GELU,
SiLU, the time features, the conditioning, tempered sampling and the
argmax rule (ties lowest, NaN never wins) by closed forms.  The
random-weight DiT as a whole has no printed values on the pages to pin it
to, so its numeric identity with the authors' trained model is "parity
unpinned": only its parts and the two independent formulations agree.
"""
