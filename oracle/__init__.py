"""CPU oracle for the paged INT4/INT8-protected KV cache and its decode attention.

THIS PACKAGE IS TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import, call or execute anything
in it.  The product path (the CUDA library and its Python binding) never
imports it and never falls back to it.

It is a plain, slow restatement of what the method computes, written from the
two pages that define it:

* "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
  Serving", Abstract: token-wise INT4 quantization of K/V after a
  block-diagonal Hadamard rotation, written by a fused rotate-quantize step
  straight into a paged KV-cache layout, consumed by fused decode attention.
* "KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4 KV Cache
  Quantization", Abstract: calibration-free INT4 KV with selective INT8
  protection of a bounded set of positions (attention sinks plus the recent
  context).

Arithmetic: the rotation and the quantizer run in fp32 with a fixed operation
order (so packed codes can be compared bit for bit), attention runs in fp64.
Modules:

* ``hadamard``  -- Sylvester Hadamard matrix (closed form) and the fp32 FWHT.
* ``quant``     -- fp16 directed rounding, the asymmetric token-wise quantizer.
* ``layout``    -- byte placement of codes and scales inside a 16-token tile.
* ``cache``     -- the paged cache: block table, INT4 pages, INT8 sink/ring
                  store, append and the effective (dequantized) view.
* ``attention`` -- fp64 GQA decode attention over the effective view, and the
                  causal attention of several query tokens per sequence.

Parity unpinned: none of the functions here lacks a pin; the end-to-end
accuracy effect of INT4 versus BF16 (a model-level claim of both pages) is out
of scope because it needs trained weights and datasets.
"""

from . import hadamard, quant, layout, cache, attention, rope  # noqa: F401
from .hadamard import sylvester_hadamard, block_diag_hadamard, fwht_fp32, rotation_constant_fp32  # noqa: F401
from .quant import (quantize_groups, dequantize_groups, fp16_round_down, fp16_round_up,  # noqa: F401
                    bf16_round, clamp_fp16_range)
from .cache import OracleKV4Cache, OracleBF16Cache, prot_slot, n_prot_tiles  # noqa: F401
from .attention import attention_fp64, decode_attention, decode_attention_bf16, extend_attention  # noqa: F401
from .rope import rope_fp32, NEOX as ROPE_NEOX, GPTJ as ROPE_GPTJ  # noqa: F401
