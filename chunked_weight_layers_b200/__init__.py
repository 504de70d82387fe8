"""B200-native fast-weight (test-time-training) chunk scan.

The work happens in libttt.so (hand-written CUDA for sm_100a behind a C ABI, declared in
include/ttt.h). This module is its thin Python binding: :class:`FastWeightState` turns
torch tensors into device pointers and the current CUDA stream and calls the C entry
points of the same names. There is no CPU or PyTorch fallback: without the compiled
library, or without a CUDA device, every call raises.
"""

from __future__ import annotations

import ctypes

from . import abi
from .abi import TTTError, check  # noqa: F401

__all__ = ["FastWeightState", "TTTError", "config", "abi"]


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def _current_raw_stream():
    """A function returning torch's current CUDA stream handle of the current device: torch's
    direct accessor when present (a fraction of a microsecond a call), else the public API."""
    import torch
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    cur_dev = getattr(torch._C, "_cuda_getDevice", None)
    if raw is not None and cur_dev is not None:
        return lambda: raw(cur_dev())
    return lambda: torch.cuda.current_stream().cuda_stream


_raw_stream = None


def _stream(stream) -> int | None:
    global _raw_stream
    if stream is None:
        if _raw_stream is None:
            _raw_stream = _current_raw_stream()
        return _raw_stream() or None
    return stream.cuda_stream or None


def config(rule: str, **fields) -> abi.ttt_config:
    """A ttt_config with the library's defaults for ``rule`` ("inplace" or "linear"), then
    ``fields`` applied (e.g. ``d_key=512, d_val=256, chunk=512, eta=0.01, io_dtype=0``)."""
    lib = abi.load()
    cfg = abi.ttt_config()
    r = abi.TTT_RULE_INPLACE_HEBBIAN if rule == "inplace" else abi.TTT_RULE_LINEAR_GD
    check(lib.ttt_config_init(ctypes.byref(cfg), r))
    for k, v in fields.items():
        if not hasattr(cfg, k):
            raise AttributeError(k)
        setattr(cfg, k, v)
    return cfg


class FastWeightState:
    """Owner of one ttt_state (device weights, gate threshold and residual cache)."""

    def __init__(self, cfg: abi.ttt_config, W0, Wtarget=None, convw=None, stream=None):
        self._lib = abi.load()
        self.cfg = cfg
        h = ctypes.c_void_p()
        check(self._lib.ttt_state_create(ctypes.byref(cfg), _ptr(W0), _ptr(Wtarget), _ptr(convw),
                                         _stream(stream), ctypes.byref(h)))
        self._h = h

    @property
    def handle(self) -> int:
        return self._h.value

    def chunk_scan(self, keys, targets, queries=None, out=None, loss_out=None, T=None, stream=None):
        """ttt_chunk_scan on device tensors; ``T`` defaults to the token dimension of keys."""
        if T is None:
            T = keys.shape[-2]
        check(self._lib.ttt_chunk_scan(self._h, _ptr(keys), _ptr(targets), _ptr(queries), int(T),
                                       _ptr(out), _ptr(loss_out), _stream(stream)))

    def chunk_scan_host(self, keys, targets, queries=None, out=None, loss_out=None, T=None, stream=None):
        """ttt_chunk_scan_host on CPU tensors (pinned for full speed); synchronises."""
        if T is None:
            T = keys.shape[-2]
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        check(self._lib.ttt_chunk_scan_host(self._h, p(keys), p(targets), p(queries), int(T), p(out),
                                            p(loss_out), _stream(stream)))

    def surprisal_route(self, loss, T=None, stream=None):
        if T is None:
            T = loss.shape[-1]
        check(self._lib.ttt_surprisal_route(self._h, _ptr(loss), int(T), _stream(stream)))

    def reset(self, stream=None):
        check(self._lib.ttt_state_reset(self._h, _stream(stream)))

    def get_weights(self, W, stream=None):
        check(self._lib.ttt_state_get_weights(self._h, _ptr(W), _stream(stream)))
        return W

    def set_weights(self, W, stream=None):
        check(self._lib.ttt_state_set_weights(self._h, _ptr(W), _stream(stream)))

    def cache_read(self, entries=None, counts=None, stream=None):
        check(self._lib.ttt_cache_read(self._h, _ptr(entries), _ptr(counts), _stream(stream)))

    def gate_read(self, tau=None, tau_set=None, stream=None):
        check(self._lib.ttt_gate_read(self._h, _ptr(tau), _ptr(tau_set), _stream(stream)))

    def poll(self):
        check(self._lib.ttt_state_poll(self._h))

    def launch_count(self) -> int:
        return int(self._lib.ttt_state_launch_count(self._h))

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            check(self._lib.ttt_state_destroy(self._h))
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
