"""The C-ABI library without a GPU: it loads, exports every entry point the
headers declare, and rejects invalid configurations and arguments on the host
(no kernel is launched)."""
import ctypes
import os
import re

import pytest

from compact_decode_attention_b200 import build as dbuild
from compact_decode_attention_b200 import dms

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dbuild.build()
    return dms.lib()


def declared_entry_points():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(dms_\w+)\s*\(", src, flags=re.M))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(dms.EXPORTED), "binding and headers disagree"


def test_status_strings(lib):
    assert dms.dms_status_string(dms.DMS_OK) == "DMS_OK"
    assert dms.dms_status_string(dms.DMS_ERR_DEVICE) == "DMS_ERR_DEVICE"


def cfg(**kw):
    base = dict(n_layers=36, max_batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, window=512,
                block_tokens=64, kv_dtype=dms.DMS_BF16, max_blocks=10000, max_context=8192 + 129)
    base.update(kw)
    return dms.PoolConfig(**base)


def test_pool_bytes_cover_blocks_and_tables(lib):
    c = cfg()
    n = dms.dms_pool_bytes_required(c)
    assert n >= 10000 * 2 * 64 * 128 * 2
    assert n % 256 == 0


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), dms.DMS_ERR_UNSUPPORTED),
    (dict(n_q_heads=30), dms.DMS_ERR_INVALID_ARG),
    (dict(n_q_heads=128), dms.DMS_ERR_UNSUPPORTED),
    (dict(block_tokens=32), dms.DMS_ERR_UNSUPPORTED),
    (dict(kv_dtype=7), dms.DMS_ERR_INVALID_ARG),
    (dict(window=0), dms.DMS_ERR_INVALID_ARG),
    (dict(kv_dtype=dms.DMS_FP8_E4M3, head_dim=64), dms.DMS_ERR_UNSUPPORTED),
    (dict(max_context=1 << 24), dms.DMS_ERR_INVALID_ARG),
])
def test_invalid_configs_rejected(lib, bad, status):
    with pytest.raises(dms.DmsError) as e:
        dms.dms_pool_bytes_required(cfg(**bad))
    assert e.value.status == status


def test_null_arguments_rejected_without_cuda(lib):
    out = ctypes.c_void_p()
    assert lib.dms_pool_create(ctypes.byref(cfg()), None, 1 << 30, None, ctypes.byref(out)) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_pool_stats(None, None, None) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_compact_prefill(None, 0, 1, 1, None, None, 1, None, None) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_decode_attn(None, 0, 1, None, 1, None, 0.0, None, 0, None) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_synth_normal(0, 0, 0, 1, 1, 0, 1, 1, 64, 1, None, None) == dms.DMS_ERR_INVALID_ARG
    # host settings of a pool handle
    assert lib.dms_pool_set_prefill_mode(None, dms.PREFILL_SPARSE) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_pool_set_attn_kernel(None, dms.ATTN_AUTO) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_pool_set_wait_limit(None, 1000000) == dms.DMS_ERR_INVALID_ARG
    assert lib.dms_last_error().decode()


def test_product_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(dms, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(dms, "_lib", None)
    with pytest.raises(dms.DmsLibraryMissing):
        dms.lib()
