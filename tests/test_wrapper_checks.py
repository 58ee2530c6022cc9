"""The owning wrappers refuse, before anything is launched, a tensor argument the
kernels would misread (wrong device, dtype or layout, or too few elements for the
call).  `need` looks only at tensor metadata, so CPU tensors exercise it here."""

import pytest
import torch

kv4 = pytest.importorskip("int4_kv_cache_paged_b200")
from int4_kv_cache_paged_b200.cache import need, _out_dtypes  # noqa: E402

CPU = torch.device("cpu")
BF16 = (torch.bfloat16,)


def _refused(*args):
    with pytest.raises(kv4.KV4Error) as e:
        need(*args)
    assert e.value.code == kv4.KV4_ERR_INVALID_ARG
    return str(e.value)


def test_a_fitting_tensor_passes():
    need(torch.zeros(4, 8, 64, dtype=torch.bfloat16), "q", BF16, 4 * 8 * 64, CPU)
    need(torch.zeros(5, 8, 64, dtype=torch.bfloat16), "q", BF16, 4 * 8 * 64, CPU)     # more rows than read
    need(torch.zeros(3, dtype=torch.int64), "workspace", None, 0, CPU)                 # any dtype
    need(torch.zeros(0, dtype=torch.bfloat16), "k_new", BF16, 0, CPU)


def test_each_mismatch_is_refused():
    msg = _refused(torch.zeros(4, 8, 64, dtype=torch.float16), "q", BF16, 4 * 8 * 64, CPU)
    assert "q must be" in msg and "float16" in msg
    _refused(torch.zeros(4, 8, 64, dtype=torch.bfloat16), "q", BF16, 5 * 8 * 64, CPU)         # too small
    msg = _refused(torch.zeros(64, 8, dtype=torch.bfloat16).t(), "q", BF16, 8 * 64, CPU)      # strided
    assert "not contiguous" in msg
    _refused(torch.zeros(8, dtype=torch.int32), "seq_ids", (torch.int32,), 8, torch.device("cuda", 0))
    _refused([0, 1, 2], "seq_ids", (torch.int32,), 3, CPU)
    _refused(torch.zeros(8, dtype=torch.int64), "cu_new", (torch.int32,), 8, CPU)


def test_output_dtype_follows_the_mode():
    assert _out_dtypes(0) == (torch.bfloat16,)
    assert _out_dtypes(kv4.KV4_MODE_OUT_F32) == (torch.float32,)
    assert _out_dtypes(kv4.KV4_MODE_OUT_F32 | kv4.KV4_MODE_INT4_ONLY) == (torch.float32,)
