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
    for rule in (abi.TTT_RULE_LINEAR_LN_GD, abi.TTT_RULE_MLP_GD):
        assert lib.ttt_config_init(ctypes.byref(cfg), rule) == abi.TTT_OK
        assert (cfg.rule, cfg.chunk, cfg.d_key, cfg.d_val, cfg.io_dtype) == (rule, 16, 64, 64, abi.TTT_BF16)
        assert cfg.ln_eps == ctypes.c_float(1e-6).value
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
    assert lib.ttt_chunk_scan_packed(None, None, None, None, 0, None, None, None, None, None) == abi.TTT_ERR_INVALID_ARG
    assert lib.ttt_state_set_layernorm(None, None, None, None) == abi.TTT_ERR_INVALID_ARG
    assert lib.ttt_state_destroy(None) == abi.TTT_OK
    assert lib.ttt_state_launch_count(None) == 0
    assert lib.ttt_abi_version() == 2


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


def test_binding_checks_buffers_before_any_call():
    """The binding's per-tensor check (element type, element count, contiguity, device) runs
    before the C call and names the offending argument; host tensors pass only where a host
    buffer is expected."""
    import torch
    from chunked_weight_layers_b200 import _arg
    t = torch.zeros(4, 16, dtype=torch.bfloat16)
    assert _arg(None, "x", torch.bfloat16, 64, None) is None
    assert _arg(t, "keys", torch.bfloat16, 64, None) == t.data_ptr()
    assert _arg(t, "keys", torch.bfloat16, 32, None) == t.data_ptr()  # larger buffers are fine
    with pytest.raises(ValueError, match="keys: .*at least 65 elements"):
        _arg(t, "keys", torch.bfloat16, 65, None)
    with pytest.raises(ValueError, match="targets: .*torch.float32"):
        _arg(t, "targets", torch.float32, 64, None)
    with pytest.raises(ValueError, match="not contiguous"):
        _arg(t.t(), "out", torch.bfloat16, 64, None)
    with pytest.raises(ValueError, match="on cuda:0, got .* on cpu"):
        _arg(t, "keys", torch.bfloat16, 64, 0)


def test_binding_element_counts_follow_the_config(monkeypatch):
    """The counts the binding demands are those include/ttt.h states for each rule's buffers."""
    import torch
    import chunked_weight_layers_b200 as cwl
    seen = {}

    def fake_arg(t, name, dtype, numel, dev):
        seen[name] = (dtype, numel)
        return None

    monkeypatch.setattr(cwl, "_arg", fake_arg)
    cases = [
        # TTT-Linear, B=2, H=3, gate on with 8 cache entries, T=64: [B,H,T,64] io, [B,H,T] loss.
        (dict(rule=1, io_dtype=1, batch=2, heads=3, d_key=64, d_val=64, chunk=16, gate_enable=1,
              cache_capacity=8), 64,
         dict(keys=24576, targets=24576, queries=24576, out=24576, loss_out=384), 24576, 8),
        # TTT-Linear without the gate: the library keeps a one-entry cache per pair.
        (dict(rule=1, io_dtype=1, batch=1, heads=5, d_key=64, d_val=64, chunk=16, gate_enable=0,
              cache_capacity=256), 32,
         dict(keys=10240, targets=10240, queries=10240, out=10240, loss_out=160), 20480, 1),
        # In-Place bf16, f=512, d=256, T=384: Z [T,f], V̂ or X0 [T,d], O [T,d], W [d,f].
        (dict(rule=0, io_dtype=1, batch=1, heads=1, d_key=512, d_val=256, chunk=128), 384,
         dict(keys=196608, targets=98304, out=98304), 131072, 1),
        # In-Place fp32 with the same widths.
        (dict(rule=0, io_dtype=0, batch=1, heads=1, d_key=512, d_val=256, chunk=128), 384,
         dict(keys=196608, targets=98304, out=98304), 131072, 1),
        # TTT-Linear with LayerNorm, B=1, H=2, T=32: W [B,H,64,64].
        (dict(rule=2, io_dtype=1, batch=1, heads=2, d_key=64, d_val=64, chunk=16), 32,
         dict(keys=4096, targets=4096, queries=4096, out=4096, loss_out=64), 8192, 1),
        # TTT-MLP, B=1, H=2: W1 [64, 256] and W2 [256, 64] per pair.
        (dict(rule=3, io_dtype=1, batch=1, heads=2, d_key=64, d_val=64, chunk=16), 32,
         dict(keys=4096, targets=4096, queries=4096, out=4096, loss_out=64), 65536, 1),
    ]
    for fields, T, want, nW, cap in cases:
        cfg = cwl.abi.ttt_config(**fields)
        st = object.__new__(cwl.FastWeightState)
        st._inplace, st._io, st._bh, st._dk, st._dv, st._nW, st._cap = cwl._layout(cfg)
        assert (st._nW, st._cap) == (nW, cap)
        seen.clear()
        st._scan_args(None, None, None, None, None, T, 0)
        io = torch.float32 if fields["io_dtype"] == 0 else torch.bfloat16
        for name, n in want.items():
            assert seen[name] == (torch.float32 if name == "loss_out" else io, n), (fields, name)
