"""B200-native fast-weight (test-time-training) chunk scan.

The work happens in libttt.so (hand-written CUDA for sm_100a behind a C ABI, declared in
include/ttt.h). This module is its thin Python binding: :class:`FastWeightState` turns
torch tensors into device pointers and the current CUDA stream and calls the C entry
points of the same names. There is no CPU or PyTorch fallback: without the compiled
library, or without a CUDA device, every call raises.

The C ABI takes bare pointers, so it cannot see a buffer's size or element type. Before each
call the binding checks what only it can see: every tensor has the element type and at
least the element count the call reads or writes (from the state's configuration and T),
is contiguous, and lives on the current CUDA device. A tensor that fails raises ValueError
and nothing is launched; everything else (T against the chunk, which buffers a rule takes,
alignment) is the library's to reject.
"""

from __future__ import annotations

import ctypes

import torch

from . import abi
from .abi import TTTError, check  # noqa: F401

__all__ = ["FastWeightState", "TTTError", "config", "abi"]


# torch's current CUDA device of this thread (its direct accessor when present: it is called
# on every scan).
_current_device = getattr(torch._C, "_cuda_getDevice", None) or torch.cuda.current_device


def _arg(t, name: str, dtype, numel: int, dev: int | None) -> int | None:
    """Device (or, with ``dev`` None, host) address of ``t`` once it is known to hold at
    least ``numel`` contiguous elements of ``dtype`` on device ``dev``."""
    if t is None:
        return None
    if (t.dtype is not dtype or t.numel() < numel or not t.is_contiguous()
            or (t.get_device() != dev if dev is not None else t.is_cuda)):
        where = "the host" if dev is None else f"cuda:{dev}"
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor of at least {numel} elements on "
                         f"{where}, got {tuple(t.shape)} {t.dtype} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")
    return t.data_ptr()


def _current_raw_stream():
    """A function returning torch's current CUDA stream handle of the current device: torch's
    direct accessor when present (a fraction of a microsecond a call), else the public API."""
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


RULES = {"inplace": abi.TTT_RULE_INPLACE_HEBBIAN, "linear": abi.TTT_RULE_LINEAR_GD,
         "linear_ln": abi.TTT_RULE_LINEAR_LN_GD, "mlp": abi.TTT_RULE_MLP_GD}


def add_f32(y, x, alpha: float = 1.0, stream=None):
    """ttt_add_f32: y ← y + alpha·x for fp32 device tensors of the same size; returns y."""
    dev = _current_device()
    n = y.numel()
    check(abi.load().ttt_add_f32(_arg(y, "y", torch.float32, n, dev), _arg(x, "x", torch.float32, n, dev),
                                 float(alpha), n, _stream(stream)))
    return y


def config(rule: str, **fields) -> abi.ttt_config:
    """A ttt_config with the library's defaults for ``rule`` ("inplace", "linear", "linear_ln"
    or "mlp"), then ``fields`` applied (e.g. ``d_key=512, d_val=256, chunk=512, eta=0.01``)."""
    lib = abi.load()
    cfg = abi.ttt_config()
    r = RULES[rule]
    check(lib.ttt_config_init(ctypes.byref(cfg), r))
    for k, v in fields.items():
        if not hasattr(cfg, k):
            raise AttributeError(k)
        setattr(cfg, k, v)
    return cfg


def _layout(cfg: abi.ttt_config):
    """(In-Place?, io element type, sequence-head pairs, d_key, d_val, weight elements, cache
    entries per pair) of a state created with ``cfg``, as include/ttt.h lays its buffers out."""
    inplace = cfg.rule == abi.TTT_RULE_INPLACE_HEBBIAN
    io = torch.float32 if cfg.io_dtype == abi.TTT_F32 else torch.bfloat16
    bh = 1 if inplace else cfg.batch * cfg.heads
    nW = cfg.d_val * cfg.d_key if inplace else bh * cfg.d_key * cfg.d_key
    if cfg.rule == abi.TTT_RULE_MLP_GD:
        nW = bh * 2 * 64 * 256  # W1 [64, 256] then W2 [256, 64] per (sequence, head)
    cap = cfg.cache_capacity if (not inplace and cfg.gate_enable) else 1
    return inplace, io, bh, cfg.d_key, cfg.d_val, nW, cap


class FastWeightState:
    """Owner of one ttt_state (device weights, gate threshold and residual cache)."""

    def __init__(self, cfg: abi.ttt_config, W0, Wtarget=None, convw=None, stream=None):
        self._lib = abi.load()
        self.cfg = cfg
        # Element counts the calls need, fixed at creation (the library keeps its own copy of cfg).
        self._inplace, self._io, self._bh, self._dk, self._dv, self._nW, self._cap = _layout(cfg)
        dev = _current_device()
        h = ctypes.c_void_p()
        check(self._lib.ttt_state_create(
            ctypes.byref(cfg), _arg(W0, "W0", torch.float32, self._nW, dev),
            _arg(Wtarget, "Wtarget", torch.bfloat16, cfg.d_val * cfg.d_val, dev),
            _arg(convw, "convw", torch.float32, cfg.d_val * cfg.conv_taps, dev),
            _stream(stream), ctypes.byref(h)))
        self._h = h

    @property
    def handle(self) -> int:
        return self._h.value

    def _scan_args(self, keys, targets, queries, out, loss_out, T, dev):
        io, bh = self._io, self._bh
        nk, nv = bh * T * self._dk, bh * T * self._dv
        no = T * self._dv if self._inplace else nk
        return (_arg(keys, "keys", io, nk, dev), _arg(targets, "targets", io, nv, dev),
                _arg(queries, "queries", io, nk, dev), int(T), _arg(out, "out", io, no, dev),
                _arg(loss_out, "loss_out", torch.float32, bh * T, dev))

    def chunk_scan(self, keys, targets, queries=None, out=None, loss_out=None, T=None, stream=None):
        """ttt_chunk_scan on device tensors; ``T`` defaults to the token dimension of keys."""
        if T is None:
            T = keys.shape[-2]
        check(self._lib.ttt_chunk_scan(self._h, *self._scan_args(keys, targets, queries, out, loss_out, T,
                                                                 _current_device()), _stream(stream)))

    def chunk_scan_host(self, keys, targets, queries=None, out=None, loss_out=None, T=None, stream=None):
        """ttt_chunk_scan_host on CPU tensors (pinned for full speed); synchronises."""
        if T is None:
            T = keys.shape[-2]
        check(self._lib.ttt_chunk_scan_host(self._h, *self._scan_args(keys, targets, queries, out, loss_out, T,
                                                                      None), _stream(stream)))

    def chunk_scan_docs(self, keys, targets, doc_starts, clip=None, out=None, T=None, stream=None):
        """ttt_chunk_scan_docs (In-Place BF16 states with given targets): documents laid end to
        end, ``doc_starts`` their first tokens (a sequence of ints, 0 first), each scanned from
        the pretrained weight; ``clip`` the Frobenius norm each chunk delta is clipped to (None:
        no clipping). Synchronises the stream (the layout goes up from host memory)."""
        import ctypes
        if T is None:
            T = keys.shape[-2]
        starts = (ctypes.c_int64 * len(doc_starts))(*[int(a) for a in doc_starts])
        dev = _current_device()
        check(self._lib.ttt_chunk_scan_docs(self._h, _arg(keys, "keys", self._io, T * self._dk, dev),
                                            _arg(targets, "targets", self._io, T * self._dv, dev), int(T),
                                            _arg(out, "out", self._io, T * self._dv, dev),
                                            ctypes.cast(starts, ctypes.c_void_p), len(doc_starts),
                                            float(clip or 0.0), _stream(stream)))

    def chunk_scan_packed(self, keys, targets, doc_starts, queries=None, out=None, loss_out=None, T=None,
                          stream=None):
        """ttt_chunk_scan_packed (the TTT-Linear family): ``doc_starts[b]`` lists sequence b's
        document starts (ints, 0 first); every document is scanned from the pretrained weights.
        Synchronises the stream (the layout goes up from host memory)."""
        import ctypes
        if T is None:
            T = keys.shape[-2]
        if len(doc_starts) != self.cfg.batch:
            raise ValueError(f"doc_starts must hold one list per sequence ({self.cfg.batch})")
        flat = [int(a) for seq in doc_starts for a in seq]
        starts = (ctypes.c_int64 * len(flat))(*flat)
        counts = (ctypes.c_int32 * len(doc_starts))(*[len(seq) for seq in doc_starts])
        check(self._lib.ttt_chunk_scan_packed(self._h, *self._scan_args(keys, targets, queries, out, loss_out, T,
                                                                        _current_device()),
                                              ctypes.cast(starts, ctypes.c_void_p), ctypes.cast(counts, ctypes.c_void_p),
                                              _stream(stream)))

    def surprisal_route(self, loss, T=None, stream=None):
        if T is None:
            T = loss.shape[-1]
        check(self._lib.ttt_surprisal_route(self._h, _arg(loss, "loss", torch.float32, self._bh * T, _current_device()),
                                            int(T), _stream(stream)))

    def cache_attention(self, queries, keys, values, o_ttt, alpha, out=None, T=None, stream=None):
        """ttt_cache_attention: ``out`` (default: ``o_ttt``, updated in place) = o_ttt +
        clamp(alpha, 0, 1) ⊙ the attention of each query over the cache entries it may see."""
        if T is None:
            T = keys.shape[-2]
        if out is None:
            out = o_ttt
        dev = _current_device()
        n = self._bh * T * self._dk
        check(self._lib.ttt_cache_attention(
            self._h, _arg(queries, "queries", torch.bfloat16, n, dev), _arg(keys, "keys", torch.bfloat16, n, dev),
            _arg(values, "values", torch.bfloat16, n, dev), _arg(o_ttt, "o_ttt", torch.bfloat16, n, dev),
            _arg(alpha, "alpha", torch.float32, self.cfg.heads * self._dk, dev), int(T),
            _arg(out, "out", torch.bfloat16, n, dev), _stream(stream)))
        return out

    def reset(self, stream=None):
        check(self._lib.ttt_state_reset(self._h, _stream(stream)))

    def get_weights(self, W, stream=None):
        check(self._lib.ttt_state_get_weights(self._h, _arg(W, "W", torch.float32, self._nW, _current_device()),
                                              _stream(stream)))
        return W

    def set_weights(self, W, stream=None):
        check(self._lib.ttt_state_set_weights(self._h, _arg(W, "W", torch.float32, self._nW, _current_device()),
                                              _stream(stream)))

    def set_layernorm(self, gamma, beta, stream=None):
        """ttt_state_set_layernorm: the inner model's LayerNorm gain and bias, fp32 [heads, 64]."""
        dev = _current_device()
        n = self.cfg.heads * 64
        check(self._lib.ttt_state_set_layernorm(self._h, _arg(gamma, "gamma", torch.float32, n, dev),
                                                _arg(beta, "beta", torch.float32, n, dev), _stream(stream)))

    def cache_read(self, entries=None, counts=None, stream=None):
        dev = _current_device()
        check(self._lib.ttt_cache_read(self._h, _arg(entries, "entries", torch.int32, self._bh * self._cap * 3, dev),
                                       _arg(counts, "counts", torch.int32, self._bh * 2, dev), _stream(stream)))

    def gate_read(self, tau=None, tau_set=None, stream=None):
        dev = _current_device()
        check(self._lib.ttt_gate_read(self._h, _arg(tau, "tau", torch.float32, self._bh, dev),
                                      _arg(tau_set, "tau_set", torch.int32, self._bh, dev), _stream(stream)))

    def set_option(self, option: int, value: int):
        """ttt_state_set_option (e.g. ``abi.TTT_OPT_LINEAR_CHUNK``)."""
        check(self._lib.ttt_state_set_option(self._h, int(option), int(value)))

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

