"""GPTQ layer quantization for NVIDIA B200 (sm_100a): C-ABI library + thin Python binding.

The compute path lives in ``libgptq_b200.so`` (see include/gptq_b200.h); this
package only marshals arguments.  Import fails loudly at first use when the
library has not been built (``python -m post_weight_quantization_14_b200.build``).
"""

from .gptq import (  # noqa: F401
    GPTQError,
    GptqConfig,
    LayerBuffers,
    QuantizedLayer,
    gptq_dequant,
    gptq_hessian_accumulate,
    gptq_layer_loss,
    gptq_pack_int,
    gptq_prepare_hinv,
    gptq_quantize_layer,
    gptq_selftest_bounded_wait,
    gptq_sync_status,
    gptq_timing_enable,
    gptq_timing_report,
    header_functions,
    lib,
    make_config,
    n_groups,
    quantize_layer,
)
