"""Python binding of libkv4.so: paged INT4 KV cache with INT8-protected positions, for B200.

The functions below have the names of the C ABI in include/kv4.h and only
marshal arguments (torch tensors -> device pointers, streams -> handles).
Every step of the computation runs in the CUDA library; there is no CPU or
PyTorch fallback, and importing this package fails when the library has not
been built (python int4_kv_cache_paged_b200/build.py).

Methods implemented by the library:
  "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
  Serving", Abstract (block-diagonal Hadamard + token-wise INT4 in a paged
  layout, fused rotate-quantize, fused attention) and "KV4-RL: Unlocking Faster
  Asynchronous Rollouts for RLVR with INT4 KV Cache Quantization", Abstract
  (INT8 protection of attention sinks and recent tokens).
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkv4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libkv4.so is not built: run `python int4_kv_cache_paged_b200/build.py` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)

KV4_OK = 0
KV4_ERR_INVALID_ARG = -1
KV4_ERR_UNSUPPORTED = -2
KV4_ERR_CAPACITY = -3
KV4_ERR_CUDA = -4
KV4_ERR_DEVICE_FAULT = -5
KV4_ERR_WORKSPACE = -6
KV4_ERR_SCRATCH = -7
KV4_NOALLOC_SCRATCH_BYTES = 16 << 20

KV4_DEV_BAD_PAGE = 1
KV4_DEV_OVERFLOW = 2
KV4_DEV_RANGE = 4
KV4_DEV_TIMEOUT = 8
KV4_DEV_BAD_SEQ = 16
KV4_DEV_WORKSPACE = 32
KV4_DEV_ROPE_POS = 64
KV4_DEV_BAD_CU = 128

KV4_MODE_PROTECTED = 0
KV4_MODE_INT4_ONLY = 1
KV4_MODE_OUT_F32 = 2
KV4_MODE_Q_ROTATED = 4
KV4_MODE_OUT_ROTATED = 8
KV4_MODE_ROPE_Q = 16
KV4_ROPE_NEOX = 0
KV4_ROPE_GPTJ = 1

KV4_VIEW_EFFECTIVE = 0
KV4_VIEW_INT4 = 1

KV4_FORMAT_INT4 = 0
KV4_FORMAT_NVFP4 = 1
KV4_FORMAT_INT2 = 2

EXPORTS = [
    "kv4_cache_required_bytes", "kv4_cache_create", "kv4_cache_destroy", "kv4_cache_layout", "kv4_seq_reset",
    "kv4_rotate_quantize_append", "kv4_attention_workspace_bytes", "kv4_decode_attention",
    "kv4_decode_attention_noalloc", "kv4_extend_workspace_bytes", "kv4_extend_attention",
    "kv4_set_rope", "kv4_rope_rotate_quantize_append", "kv4_decode_step",
    "kv4_dequantize_debug", "kv4_get_status", "kv4_set_attention_events", "kv4_test_stall_next_attention",
    "kv4_status_string", "kv4_version",
    "kv4bf16_cache_required_bytes", "kv4bf16_cache_create", "kv4bf16_cache_destroy", "kv4bf16_cache_layout",
    "kv4bf16_append", "kv4bf16_attention_workspace_bytes", "kv4bf16_decode_attention", "kv4bf16_get_status",
    "kv4bf16_set_attention_events",
]


class kv4_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_layers", "max_seqs", "num_q_heads", "num_kv_heads", "head_dim", "page_size", "num_pages",
        "max_pages_per_seq", "hadamard_block", "sink_tokens", "recent_window", "page_format")]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_SZ = ctypes.c_size_t
_CFG = ctypes.POINTER(kv4_config)

_sigs = {
    "kv4_cache_required_bytes": (_I, [_CFG, ctypes.POINTER(_SZ)]),
    "kv4_cache_create": (_I, [_CFG, _P, _SZ, _P, _P, ctypes.POINTER(_P)]),
    "kv4_cache_destroy": (_I, [_P]),
    "kv4_cache_layout": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "kv4_seq_reset": (_I, [_P, _I, _P]),
    "kv4_rotate_quantize_append": (_I, [_P, _I, _P, _P, _I, _I, _P, _P, _P]),
    "kv4_attention_workspace_bytes": (_I, [_P, _I, _I, ctypes.POINTER(_SZ)]),
    "kv4_decode_attention": (_I, [_P, _I, _P, _I, _P, _P, ctypes.c_float, _I, _P, _SZ, _P]),
    "kv4_decode_attention_noalloc": (_I, [_P, _I, _P, _I, _P, _P, ctypes.c_float, _I, _P]),
    "kv4_extend_workspace_bytes": (_I, [_P, _I, _I, ctypes.POINTER(_SZ)]),
    "kv4_set_rope": (_I, [_P, _P, _I, _I, _I]),
    "kv4_decode_step": (_I, [_P, _I, _P, _I, _P, _P, _P, _P, ctypes.c_float, _I, _P, _SZ, _P]),
    "kv4_rope_rotate_quantize_append": (_I, [_P, _I, _P, _P, _I, _I, _P, _P, _P]),
    "kv4_extend_attention": (_I, [_P, _I, _P, _I, _I, _P, _P, ctypes.c_float, _I, _P, _SZ, _P]),
    "kv4_dequantize_debug": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "kv4_get_status": (_I, [_P, _P, ctypes.POINTER(_I)]),
    "kv4_set_attention_events": (_I, [_P, _P, _P]),
    "kv4_test_stall_next_attention": (_I, [_P, _I]),
    "kv4bf16_set_attention_events": (_I, [_P, _P, _P]),
    "kv4_status_string": (ctypes.c_char_p, [_I]),
    "kv4_version": (ctypes.c_char_p, []),
    "kv4bf16_cache_required_bytes": (_I, [_CFG, ctypes.POINTER(_SZ)]),
    "kv4bf16_cache_create": (_I, [_CFG, _P, _SZ, _P, _P, ctypes.POINTER(_P)]),
    "kv4bf16_cache_destroy": (_I, [_P]),
    "kv4bf16_cache_layout": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "kv4bf16_append": (_I, [_P, _I, _P, _P, _I, _I, _P, _P, _P]),
    "kv4bf16_attention_workspace_bytes": (_I, [_P, _I, _I, ctypes.POINTER(_SZ)]),
    "kv4bf16_decode_attention": (_I, [_P, _I, _P, _I, _P, _P, ctypes.c_float, _I, _P, _SZ, _P]),
    "kv4bf16_get_status": (_I, [_P, _P, ctypes.POINTER(_I)]),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class KV4Error(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        super().__init__("%s: %s (%d)" % (what, _lib.kv4_status_string(code).decode(), code))


def _check(rc, what):
    if rc != KV4_OK:
        raise KV4Error(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_config(**kw):
    return kv4_config(**{k: int(v) for k, v in kw.items()})


def version():
    return _lib.kv4_version().decode()


# ---- functions with the C names (marshalling only) -------------------------

def kv4_cache_required_bytes(cfg):
    n = _SZ()
    _check(_lib.kv4_cache_required_bytes(ctypes.byref(cfg), ctypes.byref(n)), "kv4_cache_required_bytes")
    return n.value


def kv4_cache_create(cfg, buf, block_table, stream=None):
    h = _P()
    _check(_lib.kv4_cache_create(ctypes.byref(cfg), _ptr(buf), buf.numel() * buf.element_size(), _ptr(block_table),
                                 _stream(stream), ctypes.byref(h)), "kv4_cache_create")
    return h


def kv4_cache_destroy(handle):
    _check(_lib.kv4_cache_destroy(handle), "kv4_cache_destroy")


def kv4_cache_layout(handle, layer):
    pages, prot, lens = _P(), _P(), _P()
    _check(_lib.kv4_cache_layout(handle, layer, ctypes.byref(pages), ctypes.byref(prot), ctypes.byref(lens)),
           "kv4_cache_layout")
    return pages.value, prot.value, lens.value


def kv4_seq_reset(handle, seq_id, stream=None):
    _check(_lib.kv4_seq_reset(handle, seq_id, _stream(stream)), "kv4_seq_reset")


def kv4_rotate_quantize_append(handle, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, stream=None):
    _check(_lib.kv4_rotate_quantize_append(handle, layer, _ptr(seq_ids), _ptr(cu_new), n_seqs, total_new,
                                           _ptr(k_new), _ptr(v_new), _stream(stream)), "kv4_rotate_quantize_append")


def kv4_attention_workspace_bytes(handle, n_seqs, max_ctx=0):
    n = _SZ()
    _check(_lib.kv4_attention_workspace_bytes(handle, n_seqs, max_ctx, ctypes.byref(n)),
           "kv4_attention_workspace_bytes")
    return n.value


def kv4_decode_attention(handle, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, workspace, stream=None):
    _check(_lib.kv4_decode_attention(handle, layer, _ptr(seq_ids), n_seqs, _ptr(q), _ptr(out),
                                     float(softmax_scale), mode, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "kv4_decode_attention")


def kv4_decode_attention_noalloc(handle, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, stream=None):
    _check(_lib.kv4_decode_attention_noalloc(handle, layer, _ptr(seq_ids), n_seqs, _ptr(q), _ptr(out),
                                             float(softmax_scale), mode, _stream(stream)),
           "kv4_decode_attention_noalloc")


def kv4_set_rope(handle, cos_sin, max_pos, rotary_dim, style):
    _check(_lib.kv4_set_rope(handle, _ptr(cos_sin) if cos_sin is not None else None, max_pos, rotary_dim, style),
           "kv4_set_rope")


def kv4_rope_rotate_quantize_append(handle, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, stream=None):
    _check(_lib.kv4_rope_rotate_quantize_append(handle, layer, _ptr(seq_ids), _ptr(cu_new), n_seqs, total_new,
                                                _ptr(k_new), _ptr(v_new), _stream(stream)),
           "kv4_rope_rotate_quantize_append")


def kv4_decode_step(handle, layer, seq_ids, n_seqs, k_new, v_new, q, out, softmax_scale, mode, workspace,
                    stream=None):
    _check(_lib.kv4_decode_step(handle, layer, _ptr(seq_ids), n_seqs, _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(out),
                                float(softmax_scale), mode, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)),
           "kv4_decode_step")


def kv4_extend_workspace_bytes(handle, n_seqs, q_len):
    n = _SZ()
    _check(_lib.kv4_extend_workspace_bytes(handle, n_seqs, q_len, ctypes.byref(n)), "kv4_extend_workspace_bytes")
    return n.value


def kv4_extend_attention(handle, layer, seq_ids, n_seqs, q_len, q, out, softmax_scale, mode, workspace,
                         stream=None):
    _check(_lib.kv4_extend_attention(handle, layer, _ptr(seq_ids), n_seqs, q_len, _ptr(q), _ptr(out),
                                     float(softmax_scale), mode, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "kv4_extend_attention")


def kv4_dequantize_debug(handle, layer, seq_id, start, count, view, k_out, v_out, stream=None):
    _check(_lib.kv4_dequantize_debug(handle, layer, seq_id, start, count, view, _ptr(k_out), _ptr(v_out),
                                     _stream(stream)), "kv4_dequantize_debug")


def kv4_get_status(handle, stream=None):
    """Returns the device status word (and clears it)."""
    v = _I()
    rc = _lib.kv4_get_status(handle, _stream(stream), ctypes.byref(v))
    if rc not in (KV4_OK, KV4_ERR_DEVICE_FAULT):
        raise KV4Error(rc, "kv4_get_status")
    return v.value


def _event_handle(ev):
    if ev is None:
        return None
    if ev.cuda_event == 0:      # torch creates events lazily
        ev.record()
    return ctypes.c_void_p(ev.cuda_event)


def kv4_set_attention_events(handle, ev_before, ev_after):
    """ev_before / ev_after: torch.cuda.Event(enable_timing=True) or None."""
    _check(_lib.kv4_set_attention_events(handle, _event_handle(ev_before), _event_handle(ev_after)),
           "kv4_set_attention_events")


def kv4_test_stall_next_attention(handle, stage):
    """Testing hook: the next attention call's first CTA leaves `stage` unfilled (its bounded wait runs out)."""
    _check(_lib.kv4_test_stall_next_attention(handle, int(stage)), "kv4_test_stall_next_attention")


def kv4bf16_set_attention_events(handle, ev_before, ev_after):
    _check(_lib.kv4bf16_set_attention_events(handle, _event_handle(ev_before), _event_handle(ev_after)),
           "kv4bf16_set_attention_events")


def kv4bf16_cache_required_bytes(cfg):
    n = _SZ()
    _check(_lib.kv4bf16_cache_required_bytes(ctypes.byref(cfg), ctypes.byref(n)), "kv4bf16_cache_required_bytes")
    return n.value


def kv4bf16_cache_create(cfg, buf, block_table, stream=None):
    h = _P()
    _check(_lib.kv4bf16_cache_create(ctypes.byref(cfg), _ptr(buf), buf.numel() * buf.element_size(),
                                     _ptr(block_table), _stream(stream), ctypes.byref(h)), "kv4bf16_cache_create")
    return h


def kv4bf16_cache_destroy(handle):
    _check(_lib.kv4bf16_cache_destroy(handle), "kv4bf16_cache_destroy")


def kv4bf16_cache_layout(handle, layer):
    pages, lens = _P(), _P()
    _check(_lib.kv4bf16_cache_layout(handle, layer, ctypes.byref(pages), ctypes.byref(lens)), "kv4bf16_cache_layout")
    return pages.value, lens.value


def kv4bf16_append(handle, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, stream=None):
    _check(_lib.kv4bf16_append(handle, layer, _ptr(seq_ids), _ptr(cu_new), n_seqs, total_new, _ptr(k_new),
                               _ptr(v_new), _stream(stream)), "kv4bf16_append")


def kv4bf16_attention_workspace_bytes(handle, n_seqs, max_ctx=0):
    n = _SZ()
    _check(_lib.kv4bf16_attention_workspace_bytes(handle, n_seqs, max_ctx, ctypes.byref(n)),
           "kv4bf16_attention_workspace_bytes")
    return n.value


def kv4bf16_decode_attention(handle, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, workspace, stream=None):
    _check(_lib.kv4bf16_decode_attention(handle, layer, _ptr(seq_ids), n_seqs, _ptr(q), _ptr(out),
                                         float(softmax_scale), mode, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)),
           "kv4bf16_decode_attention")


def kv4bf16_get_status(handle, stream=None):
    v = _I()
    rc = _lib.kv4bf16_get_status(handle, _stream(stream), ctypes.byref(v))
    if rc not in (KV4_OK, KV4_ERR_DEVICE_FAULT):
        raise KV4Error(rc, "kv4bf16_get_status")
    return v.value


from .cache import KV4Cache, BF16Cache  # noqa: E402,F401
