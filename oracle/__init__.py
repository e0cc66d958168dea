"""CPU oracle for action-aware causal joint attention over a growing KV cache.

TEST INFRASTRUCTURE ONLY. Nothing on the product path (the C-ABI library
``libsca.so`` and its Python binding) imports, calls or links this package.
Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.

The oracle is written from the pages' prose, in plain NumPy, in float64:

* ``rule``      - token layout and the visibility rule as explicit sets of
                  visible key ranges per query (a set construction, not the
                  per-pair predicate the library uses);
* ``attention`` - dense masked softmax attention on the explicit mask;
* ``schedule``  - brute-force 128x128 tile classification from the explicit
                  mask, and the unmasked-pair count A of Eq. 6;
* ``cache``     - the growing KV cache after an append, and the descriptor
                  words the library's ABI documents;
* ``camera``    - the camera cross-attention of Eq. 3 on projected inputs
                  (visual queries over one segment's camera tokens).

Pages cited (title, section):

* [picx]   "Hy-Nomas" technical-report summary on picx.dev: Methodology >
           Model Architecture ("Segment-wise Causal Attention",
           "Action-Aware Causal Attention (Figure 6b)", "Camera-Trajectory
           Conditioning", Eq. 3); Training
           Infrastructure (Eq. 6, "Flex-Flash-Attention").
* [gpts24] "Tencent's Hy-Nomas Steers a 60-Second Video World With Text and
           Camera on One RTX 4090": "One World, Generated Segment by
           Segment" (the growing KV cache); "Inside the Architecture"
           (action-aware causal attention).
* [onedev] onedev.kr review "Hy-Nomas가 8B 모델 하나로 ...": "무엇과 다른가"
           (the head/tail split and who may see what); "어떻게 쓰나" (one
           camera token per latent frame, time-aligned cross-attention).
* [xyznot] "Hy-Nomas: Serbest Biçimli Etkileşimli Dünya Üretimine Doğru":
           "Eyleme Duyarlı Nedensel Dikkat ve Kamera Koşullandırması";
           "Dağıtık Paketleme FLOP Tahmini" (A_i of Eq. 6).

Parity pins: every function here is pinned by a ``-m "not gpu"`` test
against hand-derived visible ranges and counts (tests/golden), closed-form
counts of the unmasked pairs, a brute-force pair predicate on tiny inputs,
``torch.nn.functional.scaled_dot_product_attention``, closed-form outputs and
the invariants the pages imply. The absolute attention values have no printed
example on the pages; they rest on the library cross-check and the closed
forms.
"""
