"""Owning wrappers: device buffers allocated by torch, all work done by libkv4.so."""

import torch

from . import (make_config, kv4_cache_required_bytes, kv4_cache_create, kv4_cache_destroy, kv4_cache_layout,
               kv4_seq_reset, kv4_rotate_quantize_append, kv4_attention_workspace_bytes, kv4_decode_attention,
               kv4_decode_attention_noalloc, kv4_extend_workspace_bytes, kv4_extend_attention,
               kv4_set_rope, kv4_rope_rotate_quantize_append, kv4_decode_step, kv4_test_stall_next_attention,
               kv4_dequantize_debug, kv4_get_status, kv4bf16_cache_required_bytes, kv4bf16_cache_create,
               kv4bf16_cache_destroy, kv4bf16_cache_layout, kv4bf16_append, kv4bf16_attention_workspace_bytes,
               kv4bf16_decode_attention, kv4bf16_get_status, KV4_VIEW_EFFECTIVE, KV4_MODE_OUT_F32, KV4Error,
               KV4_ERR_INVALID_ARG)

TILE = 16
_BF16 = (torch.bfloat16,)
_I32 = (torch.int32,)


def need(t, what, dtypes, numel, device):
    """Refuse, before anything is launched, a tensor the kernels would misread: one that is not on the cache's
    device, not contiguous, of another dtype (dtypes None: any) or holding fewer elements than the call reads.
    Raises KV4Error(KV4_ERR_INVALID_ARG)."""
    if (isinstance(t, torch.Tensor) and t.device == device and t.is_contiguous()
            and (dtypes is None or t.dtype in dtypes) and t.numel() >= numel):
        return
    got = ("%s %s on %s%s" % (tuple(t.shape), t.dtype, t.device, "" if t.is_contiguous() else ", not contiguous")
           if isinstance(t, torch.Tensor) else type(t).__name__)
    raise KV4Error(KV4_ERR_INVALID_ARG, "%s must be a contiguous %s tensor of at least %d elements on %s, not %s"
                   % (what, "/".join(str(d) for d in dtypes) if dtypes else "", numel, device, got))


def _out_dtypes(mode):
    return (torch.float32,) if (mode & KV4_MODE_OUT_F32) else _BF16


def _tile4(D):
    return 16 * D + 128


def _tile8(D):
    return 32 * D + 128


def _tile16(D):
    return 64 * D


def _tilef(D):
    return 18 * D


def _tile2(D):
    return 8 * D + 128


class _Base:
    def _view(self, ptr, nbytes, shape):
        off = ptr - self.buf.data_ptr()
        return self.buf[off:off + nbytes].view(*shape)

    def seq_lens(self):
        c = self.cfg
        return self._view(self._lens_ptr, 4 * c["num_layers"] * c["max_seqs"], (-1,)).view(torch.int32).view(
            c["num_layers"], c["max_seqs"])

    def _check_rows(self, seq_ids, cu_new, k_new, v_new, total_new):
        n, dev = int(seq_ids.numel()), self.buf.device
        rows = total_new * self.cfg["num_kv_heads"] * self.cfg["head_dim"]
        if n == 0 or total_new == 0:
            return
        need(seq_ids, "seq_ids", _I32, n, dev)
        need(cu_new, "cu_new", _I32, n + 1, dev)
        need(k_new, "k_new", _BF16, rows, dev)
        need(v_new, "v_new", _BF16, rows, dev)

    def _check_attention(self, n, q_rows, q, out, mode, workspace, seq_ids):
        if n == 0:
            return
        dev, cols = self.buf.device, self.cfg["num_q_heads"] * self.cfg["head_dim"]
        need(seq_ids, "seq_ids", _I32, n, dev)
        need(q, "q", _BF16, q_rows * cols, dev)
        need(out, "out", _out_dtypes(mode), q_rows * cols, dev)
        if workspace is not None:
            need(workspace, "workspace", None, 0, dev)

    def workspace(self, n_seqs, max_ctx=0):
        nbytes = self._ws_bytes(self.handle, n_seqs, max_ctx)
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the library may already be unloaded
            pass


class KV4Cache(_Base):
    """A kv4 cache in one torch-allocated device buffer.

    cfg: dict with the kv4_config fields; block_table: int32 [max_seqs, max_pages_per_seq] (any device, copied).
    """

    def __init__(self, cfg, block_table, device="cuda", stream=None):
        self.cfg = dict(cfg)
        self.device = torch.device(device)
        self.c = make_config(**self.cfg)
        nbytes = kv4_cache_required_bytes(self.c)
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.block_table = torch.as_tensor(block_table, dtype=torch.int32).to(self.device).contiguous()
        self._ws = None
        self._ws_bytes = kv4_attention_workspace_bytes
        self.handle = kv4_cache_create(self.c, self.buf, self.block_table, stream)
        _, _, self._lens_ptr = kv4_cache_layout(self.handle, 0)

    def close(self):
        if getattr(self, "handle", None) is not None:
            kv4_cache_destroy(self.handle)
            self.handle = None

    def pages(self, layer):
        c = self.cfg
        ptr, _, _ = kv4_cache_layout(self.handle, layer)
        tile = {0: _tile4, 1: _tilef, 2: _tile2}[c.get("page_format", 0)](c["head_dim"])
        shape = (c["num_pages"], c["page_size"] // TILE, c["num_kv_heads"], tile)
        n = shape[0] * shape[1] * shape[2] * shape[3]
        return self._view(ptr, n, shape)

    def protected(self, layer):
        c = self.cfg
        _, ptr, _ = kv4_cache_layout(self.handle, layer)
        npt = -(-(c["sink_tokens"] + c["recent_window"]) // TILE)
        shape = (c["max_seqs"], npt, c["num_kv_heads"], _tile8(c["head_dim"]))
        n = shape[0] * shape[1] * shape[2] * shape[3]
        return self._view(ptr, n, shape)

    def append(self, layer, seq_ids, cu_new, k_new, v_new, total_new=None, stream=None, rope=False):
        """rope=True: each new key first gets RoPE at its position from the table of set_rope()."""
        if total_new is None:
            total_new = int(k_new.shape[0])
        self._check_rows(seq_ids, cu_new, k_new, v_new, total_new)
        fn = kv4_rope_rotate_quantize_append if rope else kv4_rotate_quantize_append
        fn(self.handle, layer, seq_ids, cu_new, int(seq_ids.numel()), total_new, k_new, v_new, stream)

    def set_rope(self, cos_sin, rotary_dim, style):
        """Register a RoPE table: fp32 [max_pos, R] on the cache's device (cos of the R/2 angles, then
        their sin); None removes it.  The cache keeps a reference to the tensor."""
        if cos_sin is None:
            kv4_set_rope(self.handle, None, 0, 0, 0)
            self._rope = None
            return
        cos_sin = cos_sin.to(device=self.device, dtype=torch.float32).contiguous()
        kv4_set_rope(self.handle, cos_sin, int(cos_sin.shape[0]), rotary_dim, style)
        self._rope = cos_sin

    def attention(self, layer, seq_ids, q, out=None, scale=0.0, mode=0, workspace=None, stream=None):
        n = int(seq_ids.numel())
        if out is None:
            dt = torch.float32 if (mode & KV4_MODE_OUT_F32) else torch.bfloat16
            out = torch.empty(q.shape, dtype=dt, device=self.device)
        if workspace is None:
            workspace = self.workspace(n)
        self._check_attention(n, n, q, out, mode, workspace, seq_ids)
        kv4_decode_attention(self.handle, layer, seq_ids, n, q, out, scale, mode, workspace, stream)
        return out

    def decode_step(self, layer, seq_ids, k_new, v_new, q, out=None, scale=0.0, mode=0, workspace=None, stream=None):
        """Append one token per sequence (k_new, v_new [n, Hkv, D] bf16) and attend q [n, Hq, D] in one call."""
        n = int(seq_ids.numel())
        if out is None:
            dt = torch.float32 if (mode & KV4_MODE_OUT_F32) else torch.bfloat16
            out = torch.empty(q.shape, dtype=dt, device=self.device)
        if workspace is None:
            workspace = self.workspace(n)
        self._check_attention(n, n, q, out, mode, workspace, seq_ids)
        if n:
            rows = n * self.cfg["num_kv_heads"] * self.cfg["head_dim"]
            need(k_new, "k_new", _BF16, rows, self.buf.device)
            need(v_new, "v_new", _BF16, rows, self.buf.device)
        kv4_decode_step(self.handle, layer, seq_ids, n, k_new, v_new, q, out, scale, mode, workspace, stream)
        return out

    def extend_workspace(self, n_seqs, q_len):
        nbytes = kv4_extend_workspace_bytes(self.handle, n_seqs, q_len)
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    def extend_attention(self, layer, seq_ids, q, out=None, scale=0.0, mode=0, workspace=None, stream=None):
        """Attention of the last q.shape[1] positions of every sequence, each causal over the cache.

        q: bf16 [n_seqs, q_len, Hq, D]; returns out of the same shape (fp32 with KV4_MODE_OUT_F32)."""
        n, q_len = int(seq_ids.numel()), int(q.shape[1])
        if out is None:
            dt = torch.float32 if (mode & KV4_MODE_OUT_F32) else torch.bfloat16
            out = torch.empty(q.shape, dtype=dt, device=self.device)
        if workspace is None:
            workspace = self.extend_workspace(n, q_len)
        self._check_attention(n, n * q_len, q, out, mode, workspace, seq_ids)
        kv4_extend_attention(self.handle, layer, seq_ids, n, q_len, q, out, scale, mode, workspace, stream)
        return out

    def attention_noalloc(self, layer, seq_ids, q, out, scale=0.0, mode=0, stream=None):
        """Attention with the library's static scratch (no workspace); `out` must be given."""
        n = int(seq_ids.numel())
        self._check_attention(n, n, q, out, mode, None, seq_ids)
        kv4_decode_attention_noalloc(self.handle, layer, seq_ids, int(seq_ids.numel()), q, out, scale, mode, stream)
        return out

    def stall_next_attention(self, stage):
        """Testing hook: the next attention call's first CTA leaves its stage `stage` unfilled, so its bounded
        wait runs out (KV4_DEV_TIMEOUT); see kv4_test_stall_next_attention in kv4.h."""
        kv4_test_stall_next_attention(self.handle, stage)

    def dequantize(self, layer, seq, start, count, view=KV4_VIEW_EFFECTIVE, stream=None):
        c = self.cfg
        k = torch.empty((count, c["num_kv_heads"], c["head_dim"]), dtype=torch.float32, device=self.device)
        v = torch.empty_like(k)
        kv4_dequantize_debug(self.handle, layer, seq, start, count, view, k, v, stream)
        return k, v

    def reset(self, seq, stream=None):
        kv4_seq_reset(self.handle, seq, stream)

    def status(self, stream=None):
        return kv4_get_status(self.handle, stream)


class BF16Cache(_Base):
    """The BF16 baseline cache (same paging and attention structure, no quantization)."""

    def __init__(self, cfg, block_table, device="cuda", stream=None):
        self.cfg = dict(cfg)
        self.device = torch.device(device)
        self.c = make_config(**self.cfg)
        nbytes = kv4bf16_cache_required_bytes(self.c)
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.block_table = torch.as_tensor(block_table, dtype=torch.int32).to(self.device).contiguous()
        self._ws = None
        self._ws_bytes = kv4bf16_attention_workspace_bytes
        self.handle = kv4bf16_cache_create(self.c, self.buf, self.block_table, stream)
        _, self._lens_ptr = kv4bf16_cache_layout(self.handle, 0)

    def close(self):
        if getattr(self, "handle", None) is not None:
            kv4bf16_cache_destroy(self.handle)
            self.handle = None

    def pages(self, layer):
        c = self.cfg
        ptr, _ = kv4bf16_cache_layout(self.handle, layer)
        shape = (c["num_pages"], c["page_size"] // TILE, c["num_kv_heads"], _tile16(c["head_dim"]))
        n = shape[0] * shape[1] * shape[2] * shape[3]
        return self._view(ptr, n, shape)

    def append(self, layer, seq_ids, cu_new, k_new, v_new, total_new=None, stream=None):
        if total_new is None:
            total_new = int(k_new.shape[0])
        self._check_rows(seq_ids, cu_new, k_new, v_new, total_new)
        kv4bf16_append(self.handle, layer, seq_ids, cu_new, int(seq_ids.numel()), total_new, k_new, v_new, stream)

    def attention(self, layer, seq_ids, q, out=None, scale=0.0, mode=0, workspace=None, stream=None):
        n = int(seq_ids.numel())
        if out is None:
            dt = torch.float32 if (mode & KV4_MODE_OUT_F32) else torch.bfloat16
            out = torch.empty(q.shape, dtype=dt, device=self.device)
        if workspace is None:
            workspace = self.workspace(n)
        self._check_attention(n, n, q, out, mode & KV4_MODE_OUT_F32, workspace, seq_ids)
        kv4bf16_decode_attention(self.handle, layer, seq_ids, n, q, out, scale, mode, workspace, stream)
        return out

    def status(self, stream=None):
        return kv4bf16_get_status(self.handle, stream)
