"""CPU oracle for the sketched linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or call anything in this package.
The product path (the C-ABI library and its Python binding) never routes
through it, and this package imports nothing from the product package.

Everything here is plain, slow and written to be checked by eye against the
definitions on the pages: "SpaLLM: Unified Compressive Adaptation of LLMs with
Sketching" (section 2.2, Eq. 1 and groups per row; section 2.3, multiple LUT
sets; section 2.4, the identity example) and the "Sketch to Adapt" OpenReview
discussion (the corrected Eq. 6 and the mapping matrix M).  The LUT update
(AdamW, SGD, the averaging of shared gradients of section 2.1) is the
textbook optimizer the pages leave unnamed.  The sketching stage that
produces the index map and the first LUTs (section 2.2: calibration Gram
matrix, weighted Lloyd's algorithm, column-by-column mapping with error
compensation) is in ``sketching_oracle``.  Floating point is
float64 throughout; fp16 LUT values and bf16 activations widen exactly.

Parity pins: every function here is pinned by a CPU test against something
other than itself (a hand-derived golden fixture, a closed form, a library
routine, an invariant, or finite differences).  No function is unpinned.
"""
from .sketch_oracle import (  # noqa: F401
    row_stride_bytes, packed_bytes, pack, unpack, dequant, sketch_matrix,
    dequant_via_sketch_matrix, forward, backward_input, backward_lut,
    eq6_forward, eq6_backward_lut, bin_counts, trainable_params, lora_params,
    compression_factor, averaged_gradient, adamw_step, sgd_step, sketched_model_bytes,
)
from .sketching_oracle import (  # noqa: F401
    gram, damped, inverse_factor, lloyd_init, lloyd_assign, lloyd_update, lloyd,
    lloyd_luts, sketch_round, sketch_layer, proxy_loss,
)
