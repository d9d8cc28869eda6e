"""fp64 CPU oracle of the Fast-BLT local-decoder step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The CUDA
engine never calls it, shares no code with it, and fails loudly when its own
extension is missing.

What it computes, and where it is read from (page titles and sections):

* ``model``    -- one decoder pass over a set of rows: the decoder layer of
  "Fast Byte Latent Transformer (Fast-BLT) 연구 소개", section "계층적 BLT:
  인코더, 글로벌 모델, 디코더" (the one printed equation), with the attention
  masks of section "BLT-D의 어텐션 마스크" and the original byte positions for
  RoPE of section "BLT-D 학습" (block construction).
* ``policies`` -- BLT-D block decoding ("BLT-D 추론"), confidence unmasking
  ("블록 언마스킹 전략"), the greedy verification shared by BLT-S and BLT-DV
  (section "BLT-S와 BLT-DV"), BLT-S drafting ("BLT-S"), BLT-DV drafting
  ("BLT-DV"), plain greedy AR decoding, pass counters and the proxy
  memory-bandwidth formula (restated on the wangzhan123.com page, section
  "六、测量效能之方式").

Readings where the pages are silent: a SwiGLU FFN, pre-norm RMSNorm with eps
1e-5, rotate-half RoPE with theta 1e4, ``conf >= alpha``, argmax ties to the
lowest byte and fallback ties to the lowest position, and open patches seeing
the newest closed latent.  The decoder-layer
internals (RMSNorm, SwiGLU, RoPE) follow those readings: the pages fix none of
them, so their parity against the pages is unpinned; the tests pin the oracle's
implementation of each against library routines and closed-form invariants,
and the whole pass against a second statement in torch fp64
(``tests/test_oracle_restatement.py``).
"""
