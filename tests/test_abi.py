"""CPU checks of the C ABI: the library loads, exports every function include/kv4.h declares,
and rejects bad arguments before touching a device."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kv4.h")
LIB = os.path.join(ROOT, "int4_kv_cache_paged_b200", "libkv4.so")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(kv4\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.fail("libkv4.so is missing; __graft_entry__.build() must run first")
    return ctypes.CDLL(LIB)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("kv4_cache_create", "kv4_rotate_quantize_append", "kv4_decode_attention", "kv4_dequantize_debug"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert missing == []


def test_binding_names_match_header():
    import int4_kv_cache_paged_b200 as kv4
    for n in _declared():
        assert n in kv4.EXPORTS and callable(getattr(kv4, n, None) or getattr(kv4._lib, n)), n


def test_host_side_validation_without_a_device():
    import int4_kv_cache_paged_b200 as kv4
    good = dict(num_layers=1, max_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=16, num_pages=10,
                max_pages_per_seq=5, hadamard_block=128, sink_tokens=4, recent_window=16)
    n = kv4.kv4_cache_required_bytes(kv4.make_config(**good))
    # state 256 + seq_lens (256) + pool 10*2*1*2176 + INT8 store 2*2*2*4224, each rounded to 256
    pool = ((10 * 2 * 2176 + 255) // 256) * 256
    prot = ((2 * 2 * 2 * 4224 + 255) // 256) * 256
    assert n == 256 + 256 + pool + prot
    for bad, code in ((dict(head_dim=96), kv4.KV4_ERR_UNSUPPORTED), (dict(num_q_heads=7), kv4.KV4_ERR_INVALID_ARG),
                      (dict(num_q_heads=32, num_kv_heads=2), kv4.KV4_ERR_UNSUPPORTED),
                      (dict(page_size=24), kv4.KV4_ERR_UNSUPPORTED), (dict(hadamard_block=3), kv4.KV4_ERR_INVALID_ARG),
                      (dict(hadamard_block=256), kv4.KV4_ERR_INVALID_ARG), (dict(recent_window=0), kv4.KV4_ERR_INVALID_ARG),
                      (dict(sink_tokens=-1), kv4.KV4_ERR_INVALID_ARG), (dict(num_pages=0), kv4.KV4_ERR_INVALID_ARG),
                      (dict(page_format=3), kv4.KV4_ERR_INVALID_ARG), (dict(page_format=-1), kv4.KV4_ERR_INVALID_ARG)):
        with pytest.raises(kv4.KV4Error) as e:
            kv4.kv4_cache_required_bytes(kv4.make_config(**dict(good, **bad)))
        assert e.value.code == code, bad
    # NVFP4 pages: 18*D bytes per 16-token tile (the INT8 store is the same)
    nf = kv4.kv4_cache_required_bytes(kv4.make_config(**dict(good, page_format=kv4.KV4_FORMAT_NVFP4)))
    assert nf == 256 + 256 + ((10 * 2 * 2304 + 255) // 256) * 256 + prot
    # INT2 pages: 8*D + 128 bytes per tile
    n2 = kv4.kv4_cache_required_bytes(kv4.make_config(**dict(good, page_format=kv4.KV4_FORMAT_INT2)))
    assert n2 == 256 + 256 + ((10 * 2 * 1152 + 255) // 256) * 256 + prot
    # BF16 cache ignores the quantization fields, but has one page format
    kv4.kv4bf16_cache_required_bytes(kv4.make_config(**dict(good, hadamard_block=3, recent_window=0)))
    with pytest.raises(kv4.KV4Error) as e:
        kv4.kv4bf16_cache_required_bytes(kv4.make_config(**dict(good, page_format=1)))
    assert e.value.code == kv4.KV4_ERR_INVALID_ARG
    assert kv4._lib.kv4_cache_destroy(None) == kv4.KV4_ERR_INVALID_ARG
    assert kv4._lib.kv4_status_string(kv4.KV4_ERR_WORKSPACE) == b"workspace too small"
    assert kv4.version().endswith("sm_100a")


def test_newer_entry_points_reject_bad_arguments_without_a_device():
    """The multi-token, RoPE and fused-step entry points check their arguments on the host first."""
    import int4_kv_cache_paged_b200 as kv4
    lib = kv4._lib
    size = ctypes.c_size_t()
    assert lib.kv4_extend_workspace_bytes(None, 4, 2, ctypes.byref(size)) == kv4.KV4_ERR_INVALID_ARG
    assert lib.kv4_extend_attention(None, 0, None, 1, 2, None, None, 0.0, 0, None, 0, None) == kv4.KV4_ERR_INVALID_ARG
    assert lib.kv4_set_rope(None, None, 16, 64, 0) == kv4.KV4_ERR_INVALID_ARG
    assert lib.kv4_rope_rotate_quantize_append(None, 0, None, None, 1, 1, None, None, None) == kv4.KV4_ERR_INVALID_ARG
    assert lib.kv4_decode_step(None, 0, None, 1, None, None, None, None, 0.0, 0, None, 0, None) == \
        kv4.KV4_ERR_INVALID_ARG


def test_mode_bits_of_the_binding_match_the_header():
    import int4_kv_cache_paged_b200 as kv4
    text = open(HEADER).read()
    for name in ("KV4_MODE_INT4_ONLY", "KV4_MODE_OUT_F32", "KV4_MODE_Q_ROTATED", "KV4_MODE_OUT_ROTATED",
                 "KV4_MODE_ROPE_Q", "KV4_ROPE_NEOX", "KV4_ROPE_GPTJ", "KV4_DEV_ROPE_POS"):
        m = re.search(r"\b%s\s*=\s*(\d+)" % name, text)
        assert m is not None, name
        assert getattr(kv4, name) == int(m.group(1)), name


def test_every_header_constant_has_the_same_value_in_the_binding():
    """Status codes, device status bits, modes, views, page formats and RoPE styles: each enum constant of the
    header exists in the binding with its value, and the binding defines no KV4_ constant the header lacks."""
    import int4_kv_cache_paged_b200 as kv4
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    header = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(KV4_[A-Z0-9_]+)\s*=\s*(-?\d+)", text)}
    assert len(header) >= 29          # 8 status codes, 8 device bits, 6 modes, 2 views, 3 formats, 2 RoPE styles
    for name, value in header.items():
        assert getattr(kv4, name) == value, name
    m = re.search(r"#define\s+KV4_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m and kv4.KV4_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
    binding = {n for n in dir(kv4) if re.fullmatch(r"KV4_[A-Z0-9_]+", n)}
    assert binding - set(header) == {"KV4_NOALLOC_SCRATCH_BYTES"}


def test_every_status_code_has_a_message():
    import int4_kv_cache_paged_b200 as kv4
    codes = [getattr(kv4, n) for n in dir(kv4) if n == "KV4_OK" or n.startswith("KV4_ERR_")]
    assert len(codes) == 8
    msgs = [kv4._lib.kv4_status_string(c).decode() for c in codes]
    assert "unknown status" not in msgs and len(set(msgs)) == len(msgs)
    assert kv4._lib.kv4_status_string(-99).decode() == "unknown status"


def test_every_declaration_follows_its_comment():
    """Each entry point of the header sits right after a comment block that documents it (or in a run of
    declarations that follows one, for a mirror family), so its arguments and errors are stated beside it."""
    lines = open(HEADER).read().splitlines()
    decl = re.compile(r"^(int|const char\*)\s+(kv4\w+)\(")
    for i, line in enumerate(lines):
        m = decl.match(line)
        if not m:
            continue
        j = i - 1
        while j >= 0 and ((lines[j].startswith((" ", "\t")) and not lines[j].lstrip().startswith("*"))
                          or decl.match(lines[j]) or lines[j].startswith("#define")):   # continuation, sibling
            j -= 1
        assert j >= 0 and lines[j].rstrip().endswith("*/"), m.group(2)
