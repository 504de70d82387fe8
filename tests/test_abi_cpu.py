"""Host-side checks that need no GPU: the library builds, loads and exports every entry
point include/ttt.h declares; argument checks that run before any device call."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from chunked_weight_layers_b200 import abi, build
    build.build()
    return abi.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "ttt.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "ttt_chunk_scan" in names and "ttt_surprisal_route" in names
    assert "ttt_state_create" in names and "ttt_state_reset" in names
    for n in names:
        assert hasattr(lib, n), n
    from chunked_weight_layers_b200 import abi
    assert sorted(abi.exported_symbols()) == names


def test_header_mentions_no_torch():
    text = open(os.path.join(ROOT, "include", "ttt.h")).read()
    assert "torch" not in text.lower() and "at::" not in text


def test_config_defaults(lib):
    from chunked_weight_layers_b200 import abi
    cfg = abi.ttt_config()
    assert lib.ttt_config_init(ctypes.byref(cfg), abi.TTT_RULE_LINEAR_GD) == abi.TTT_OK
    assert (cfg.chunk, cfg.gate_chunk, cfg.cache_capacity) == (16, 64, 256)
    assert abs(cfg.gate_pct - 0.95) < 1e-7 and cfg.gate_ema_old == ctypes.c_float(0.9).value
    assert cfg.gate_ema_new == ctypes.c_float(0.1).value
    assert (cfg.gate_mean_num, cfg.gate_mean_den) == (4, 5)
    assert lib.ttt_config_init(None, 0) == abi.TTT_ERR_INVALID_ARG
    assert lib.ttt_config_init(ctypes.byref(cfg), 7) == abi.TTT_ERR_INVALID_ARG
    assert b"unknown rule" in lib.ttt_last_error_string()


def test_host_argument_checks(lib):
    from chunked_weight_layers_b200 import abi
    out = ctypes.c_void_p(1234)
    assert lib.ttt_state_create(None, None, None, None, None, ctypes.byref(out)) == abi.TTT_ERR_INVALID_ARG
    assert out.value is None
    assert lib.ttt_state_create(None, None, None, None, None, None) == abi.TTT_ERR_INVALID_ARG
    assert lib.ttt_chunk_scan(None, None, None, None, 0, None, None, None) == abi.TTT_ERR_INVALID_ARG
    assert lib.ttt_surprisal_route(None, None, 0, None) == abi.TTT_ERR_INVALID_ARG
    assert lib.ttt_state_destroy(None) == abi.TTT_OK
    assert lib.ttt_state_launch_count(None) == 0
    assert lib.ttt_abi_version() == 1


def test_binding_refuses_without_library(tmp_path):
    from chunked_weight_layers_b200 import abi
    with pytest.raises(RuntimeError):
        abi.load.__wrapped__(str(tmp_path / "missing.so")) if hasattr(abi.load, "__wrapped__") else \
            _load_fresh(str(tmp_path / "missing.so"))


def _load_fresh(path):
    from chunked_weight_layers_b200 import abi
    saved = abi._lib
    abi._lib = None
    try:
        return abi.load(path)
    finally:
        abi._lib = saved
