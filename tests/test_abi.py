"""The C-ABI library builds, loads, and exports every entry point declared in
include/hq.h.  CPU only: no compute call is made."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "hq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z_0-9]+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("hq_select_vlines", "hq_pack_merge", "hq_decode_attn", "hq_prefill_attn", "hq_workspace_bytes",
              "hq_prefill_workspace_bytes", "hq_status_str", "hq_last_error", "hq_cache_validate", "hq_cache_reset",
              "hq_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from hybrid_precision_attention_b200 import build
    lib_path = build.build()
    lib = ctypes.CDLL(lib_path)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    lib.hq_abi_version.restype = ctypes.c_int32
    assert lib.hq_abi_version() == 4
    lib.hq_status_str.restype = ctypes.c_char_p
    assert lib.hq_status_str(0) == b"ok"


def test_host_validation_without_gpu():
    """Descriptor checks run on the host and need no device."""
    from hybrid_precision_attention_b200 import build
    lib = ctypes.CDLL(build.build())
    import sys
    sys.path.insert(0, ROOT)
    from hybrid_precision_attention_b200.hq import HqCacheStruct
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) & ~15
    good = HqCacheStruct(1, 32, 8, 128, 128, 500, 1024, 64, *([base] * 9))
    lib.hq_cache_validate.restype = ctypes.c_int32
    assert lib.hq_cache_validate(ctypes.byref(good)) == 0
    for field, val, want in (("D", 64, 2), ("Hq", 30, 1), ("cap", 1000, 1), ("vl_cap", 20, 1), ("rho_bp", 10001, 1),
                             ("pages", base + 4, 1), ("state", 0, 1), ("Hq", 80, 2)):
        bad = HqCacheStruct.from_buffer_copy(good)
        setattr(bad, field, val)
        assert lib.hq_cache_validate(ctypes.byref(bad)) == want, field
    # the optional page table (4-byte aligned, a non-empty pool) and running scores (16-byte aligned)
    for fields, want in (({"page_table": base + 4, "n_pages": 3}, 0), ({"page_table": base + 2, "n_pages": 3}, 1),
                         ({"page_table": base, "n_pages": 0}, 1), ({"score_acc": base + 16}, 0),
                         ({"score_acc": base + 8}, 1), ({"k_bits": 8, "v_bits": 8}, 0), ({"k_bits": 4, "v_bits": 2}, 0),
                         ({"k_bits": 2, "v_bits": 4}, 0), ({"k_bits": 8, "v_bits": 4}, 2), ({"k_bits": 3}, 1),
                         ({"v_bits": 16}, 1)):
        opt = HqCacheStruct.from_buffer_copy(good)
        for k, v in fields.items():
            setattr(opt, k, v)
        assert lib.hq_cache_validate(ctypes.byref(opt)) == want, fields
    lib.hq_workspace_bytes.restype = ctypes.c_size_t
    assert lib.hq_workspace_bytes(ctypes.byref(good), 1, 0) > 0
