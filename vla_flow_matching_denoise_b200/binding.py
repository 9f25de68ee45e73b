"""Python binding of the C ABI in include/fm_expert.h (argument marshalling only).

Every step of the denoise loop runs in the CUDA kernels of libfm_expert.so;
this module only turns numpy arrays (host memory) and torch CUDA tensors
(device memory) into pointers and back.  It raises when the shared library
is missing: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

from .synth import LAYER_KEYS, ExpertShape

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfm_expert.so")

FM_W_BF16 = 0
FM_W_FP8_E4M3 = 1
FM_W_FP8_NVFP4_GU = 2
FM_W_W8A8_E4M3 = 3

STATUS = {0: "FM_OK", 1: "FM_ERR_INVALID_ARG", 2: "FM_ERR_NOT_READY", 3: "FM_ERR_OOM",
          4: "FM_ERR_CUDA", 5: "FM_ERR_TIMEOUT", 6: "FM_ERR_UNSUPPORTED"}

# Every symbol include/fm_expert.h declares.
EXPORTS = ("fm_expert_create", "fm_set_prefix", "fm_set_prefix_varlen", "fm_set_prefix_builder",
           "fm_build_prefix", "fm_get_prefix_kv", "fm_get_nvfp4_weights", "fm_quantize_act_e4m3", "fm_denoise", "fm_velocity", "fm_time_modulation",
           "fm_trace_bytes", "fm_trace_velocity", "fm_trace_batched_bytes", "fm_trace_batched",
           "fm_get_fp8_weights", "fm_sync", "fm_test_stall",
           "fm_get_geometry", "fm_profile_denoise", "fm_profile_phases", "fm_time_modulation_noalloc",
           "fm_expert_destroy", "fm_last_error", "fm_status_string",
           "fm_abi_version")


class FmConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("action_dim", ctypes.c_int), ("chunk_len", ctypes.c_int),
                ("max_prefix", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_steps", ctypes.c_int), ("rms_eps", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("wtype", ctypes.c_int)]


_P16 = ctypes.POINTER(ctypes.c_uint16)


class FmLayerWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in LAYER_KEYS]


class FmWeights(ctypes.Structure):
    _fields_ = [("time_w1", ctypes.c_void_p), ("time_w2", ctypes.c_void_p),
                ("in_proj", ctypes.c_void_p), ("out_proj", ctypes.c_void_p),
                ("out_bias", ctypes.c_void_p), ("layers", ctypes.POINTER(FmLayerWeights))]


class FmError(RuntimeError):
    def __init__(self, call: str, status: int, text: str):
        super().__init__(f"{call} -> {STATUS.get(status, status)}: {text}")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the C-ABI library (built by vla_flow_matching_denoise_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: run `python -m vla_flow_matching_denoise_b200.build`")
    lib = ctypes.CDLL(path)
    vp, ip, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.fm_expert_create.argtypes = [ctypes.POINTER(FmConfig), ctypes.POINTER(FmWeights), ip,
                                     ctypes.POINTER(vp)]
    lib.fm_set_prefix.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ip, ip, vp]
    lib.fm_denoise.argtypes = [vp, vp, ip, ip, vp, vp]
    lib.fm_velocity.argtypes = [vp, vp, ip, ip, ip, vp, vp]
    lib.fm_time_modulation.argtypes = [vp, ip, vp, vp]
    lib.fm_trace_bytes.argtypes = [vp]
    lib.fm_trace_bytes.restype = sz
    lib.fm_trace_velocity.argtypes = [vp, vp, ip, ip, vp, vp]
    lib.fm_trace_batched_bytes.argtypes = [vp, ip]
    lib.fm_trace_batched_bytes.restype = sz
    lib.fm_trace_batched.argtypes = [vp, vp, ip, ip, ip, vp, vp]
    lib.fm_get_fp8_weights.argtypes = [vp, ip, ip, vp, vp]
    lib.fm_sync.argtypes = [vp, vp]
    lib.fm_test_stall.argtypes = [vp, ip, ctypes.c_longlong]
    lib.fm_profile_denoise.argtypes = [vp, ip, ip, ip, vp, vp]
    lib.fm_profile_phases.argtypes = [vp, ip, vp, ctypes.POINTER(sz), vp]
    lib.fm_time_modulation_noalloc.argtypes = [vp, vp, ip, ip, ip, vp, vp]
    lib.fm_set_prefix_varlen.argtypes = [vp, vp, vp, ip, vp, ip, vp]
    lib.fm_set_prefix_builder.argtypes = [vp, vp, ip]
    lib.fm_build_prefix.argtypes = [vp, vp, ip, ip, vp]
    lib.fm_get_prefix_kv.argtypes = [vp, ip, ip, vp, vp]
    lib.fm_get_nvfp4_weights.argtypes = [vp, ip, ip, vp, vp, vp]
    lib.fm_quantize_act_e4m3.argtypes = [vp, vp, ip, ip, vp, vp, vp]
    lib.fm_get_geometry.argtypes = [vp, ctypes.POINTER(ip), ctypes.POINTER(ip), ctypes.POINTER(ip)]
    lib.fm_expert_destroy.argtypes = [vp]
    lib.fm_expert_destroy.restype = sz
    lib.fm_last_error.argtypes = [vp]
    lib.fm_last_error.restype = ctypes.c_char_p
    lib.fm_status_string.argtypes = [ip]
    lib.fm_status_string.restype = ctypes.c_char_p
    lib.fm_abi_version.restype = ip
    for name in ("fm_expert_create", "fm_set_prefix", "fm_denoise", "fm_velocity",
                 "fm_time_modulation", "fm_trace_velocity", "fm_get_fp8_weights", "fm_sync",
                 "fm_test_stall", "fm_trace_batched", "fm_get_geometry", "fm_profile_denoise", "fm_profile_phases", "fm_time_modulation_noalloc",
                 "fm_set_prefix_varlen", "fm_set_prefix_builder", "fm_build_prefix", "fm_get_prefix_kv",
                 "fm_get_nvfp4_weights", "fm_quantize_act_e4m3"):
        getattr(lib, name).restype = ip
    _lib = lib
    return lib


def _ptr(a) -> Optional[int]:
    """Address of a numpy array (host) or a torch tensor (host or device)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be C-contiguous")
        return a.ctypes.data
    if hasattr(a, "data_ptr"):
        if not a.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return a.data_ptr()
    raise TypeError(f"unsupported buffer type {type(a)}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    return stream if isinstance(stream, int) else stream.cuda_stream


def make_config(shape: ExpertShape, max_prefix: Optional[int] = None, max_batch: Optional[int] = None,
                max_steps: int = 64) -> FmConfig:
    return FmConfig(shape.n_layers, shape.d_model, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                    shape.d_ff, shape.action_dim, shape.chunk_len,
                    shape.prefix_len if max_prefix is None else max_prefix,
                    shape.batch if max_batch is None else max_batch, max_steps,
                    shape.rms_eps, shape.rope_base,
                    FM_W_W8A8_E4M3 if shape.w8a8 else FM_W_FP8_NVFP4_GU if shape.nvfp4_gu
                    else FM_W_FP8_E4M3 if shape.fp8 else FM_W_BF16)


class Expert:
    """One fm_expert handle: weights copied in at construction."""

    def __init__(self, shape: ExpertShape, weights: Dict, device: int = 0,
                 max_prefix: Optional[int] = None, max_batch: Optional[int] = None,
                 max_steps: int = 64, out_bias: Optional[np.ndarray] = None):
        self.lib = load()
        self.shape = shape
        self.cfg = make_config(shape, max_prefix, max_batch, max_steps)
        layers = (FmLayerWeights * shape.n_layers)()
        for i, lw in enumerate(weights["layers"]):
            for k in LAYER_KEYS:
                setattr(layers[i], k, _ptr(lw[k]))
        bias = None if out_bias is None else np.ascontiguousarray(out_bias, dtype=np.float32)
        w = FmWeights(_ptr(weights["time_w1"]), _ptr(weights["time_w2"]), _ptr(weights["in_proj"]),
                      _ptr(weights["out_proj"]), _ptr(bias), layers)
        h = ctypes.c_void_p()
        st = self.lib.fm_expert_create(ctypes.byref(self.cfg), ctypes.byref(w), device, ctypes.byref(h))
        if st != 0:
            raise FmError("fm_expert_create", st, self.lib.fm_last_error(None).decode())
        self.h = h

    # ------------------------------------------------------------------ helpers
    def _check(self, call: str, st: int):
        if st != 0:
            raise FmError(call, st, self.lib.fm_last_error(self.h).decode())

    def close(self) -> int:
        if getattr(self, "h", None):
            n = self.lib.fm_expert_destroy(self.h)
            self.h = None
            return n
        return 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def geometry(self):
        a, b, c = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        self._check("fm_get_geometry", self.lib.fm_get_geometry(self.h, ctypes.byref(a), ctypes.byref(b),
                                                                ctypes.byref(c)))
        return a.value, b.value, c.value

    # ------------------------------------------------------------------ calls
    def set_prefix(self, k: Sequence, v: Sequence, batch: int, prefix_len: int, stream=None):
        L = self.shape.n_layers
        kp = (ctypes.c_void_p * L)(*[_ptr(x) for x in k])
        vp = (ctypes.c_void_p * L)(*[_ptr(x) for x in v])
        self._check("fm_set_prefix", self.lib.fm_set_prefix(self.h, kp, vp, batch, prefix_len, _stream(stream)))

    def set_prefix_varlen(self, k: Sequence, v: Sequence, batch: int, prefix_lens: Sequence[int], p_pad: int,
                          stream=None):
        """k[l], v[l]: [batch, p_pad, H_kv, hd] bf16 bits; request b uses its first prefix_lens[b] rows."""
        L = self.shape.n_layers
        kp = (ctypes.c_void_p * L)(*[_ptr(x) for x in k])
        vp = (ctypes.c_void_p * L)(*[_ptr(x) for x in v])
        lens = (ctypes.c_int * batch)(*[int(x) for x in prefix_lens])
        self._check("fm_set_prefix_varlen", self.lib.fm_set_prefix_varlen(self.h, kp, vp, batch, lens, p_pad,
                                                                           _stream(stream)))

    def set_prefix_builder(self, weights: Sequence, d_prefix: int):
        """weights[l] = (wk, wv): bf16 bits [H_kv * hd, d_prefix] each."""
        L = self.shape.n_layers

        class PW(ctypes.Structure):
            _fields_ = [("wk", ctypes.c_void_p), ("wv", ctypes.c_void_p)]
        arr = (PW * L)(*[PW(_ptr(wk), _ptr(wv)) for wk, wv in weights])
        self._keep_builder = weights
        self._check("fm_set_prefix_builder", self.lib.fm_set_prefix_builder(self.h, arr, d_prefix))

    def build_prefix(self, hidden: Sequence, batch: int, prefix_len: int, stream=None):
        """hidden[l]: [batch, prefix_len, d_prefix] bf16 bits (numpy or torch)."""
        L = self.shape.n_layers
        hp = (ctypes.c_void_p * L)(*[_ptr(x) for x in hidden])
        self._check("fm_build_prefix", self.lib.fm_build_prefix(self.h, hp, batch, prefix_len, _stream(stream)))

    def get_prefix_kv(self, layer: int, request: int, prefix_len: int):
        s = self.shape
        k = np.empty((prefix_len, s.n_kv_heads, s.head_dim), dtype=np.uint16)
        v = np.empty_like(k)
        self._check("fm_get_prefix_kv", self.lib.fm_get_prefix_kv(self.h, layer, request, _ptr(k), _ptr(v)))
        return k, v

    def denoise(self, x0, steps: int, out=None, stream=None):
        """x0: fp32 [B, T, A] numpy (host) or torch (device).  Returns `out`."""
        if out is None:
            out = np.empty_like(x0) if isinstance(x0, np.ndarray) else x0.new_empty(x0.shape)
        B = x0.shape[0]
        self._check("fm_denoise", self.lib.fm_denoise(self.h, _ptr(x0), B, steps, _ptr(out), _stream(stream)))
        return out

    def velocity(self, x, step_index: int, steps: int, out=None, stream=None):
        if out is None:
            out = np.empty_like(x) if isinstance(x, np.ndarray) else x.new_empty(x.shape)
        self._check("fm_velocity", self.lib.fm_velocity(self.h, _ptr(x), x.shape[0], step_index, steps,
                                                         _ptr(out), _stream(stream)))
        return out

    def time_modulation(self, steps: int, stream=None) -> np.ndarray:
        n_mod = self.shape.n_mod
        out = np.empty((steps, n_mod), dtype=np.float32)
        self._check("fm_time_modulation", self.lib.fm_time_modulation(self.h, steps, _ptr(out), _stream(stream)))
        return out

    def trace_velocity(self, x: np.ndarray, step_index: int, steps: int, stream=None) -> List[Dict]:
        s = self.shape
        n = self.lib.fm_trace_bytes(self.h) // 4
        buf = np.empty(n, dtype=np.float32)
        x = np.ascontiguousarray(x, dtype=np.float32)
        self._check("fm_trace_velocity", self.lib.fm_trace_velocity(self.h, _ptr(x), step_index, steps,
                                                                     _ptr(buf), _stream(stream)))
        T, d, F = s.chunk_len, s.d_model, s.d_ff
        qn, kn = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
        out, o = [], 0
        for _ in range(s.n_layers):
            rec = {}
            for name, w in (("h_in", d), ("q", qn), ("k", kn), ("v", kn), ("o", qn), ("h_mid", d),
                            ("u", F), ("h_out", d)):
                rec[name] = buf[o:o + T * w].reshape(T, w)
                o += T * w
            out.append(rec)
        out.append({"v": buf[o:o + T * s.action_dim].reshape(T, s.action_dim)})
        return out

    def trace_batched(self, x: np.ndarray, step_index: int, steps: int, stream=None) -> List[Dict]:
        """Per-layer intermediates of one batched velocity evaluation (see
        fm_trace_batched); x: [B, T, A].  Arrays are [B * T, width]."""
        s = self.shape
        x = np.ascontiguousarray(x, dtype=np.float32)
        B = x.shape[0]
        n = self.lib.fm_trace_batched_bytes(self.h, B) // 4
        buf = np.empty(n, dtype=np.float32)
        self._check("fm_trace_batched", self.lib.fm_trace_batched(self.h, _ptr(x), B, step_index, steps,
                                                                   _ptr(buf), _stream(stream)))
        M, d, F = B * s.chunk_len, s.d_model, s.d_ff
        qn, kn = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
        out, o = [], 0
        for _ in range(s.n_layers):
            rec = {}
            for name, w in (("h_in", d), ("y_a", d), ("q", qn), ("k", kn), ("v", kn), ("o", qn),
                            ("h_mid", d), ("y_f", d), ("u", F), ("h_out", d)):
                rec[name] = buf[o:o + M * w].reshape(M, w)
                o += M * w
            out.append(rec)
        out.append({"v": buf[o:o + M * s.action_dim].reshape(M, s.action_dim)})
        return out

    def get_fp8_weights(self, layer: int, which: int, rows: int, cols: int):
        codes = np.empty((rows, cols), dtype=np.uint8)
        scale = np.empty(rows, dtype=np.float32)
        self._check("fm_get_fp8_weights", self.lib.fm_get_fp8_weights(self.h, layer, which, _ptr(codes),
                                                                       _ptr(scale)))
        return codes, scale

    def get_nvfp4_weights(self, layer: int, which: int, rows: int, cols: int):
        """(codes [rows, cols] one E2M1 code per byte, block scales [rows, cols/16] E4M3, g)."""
        codes = np.empty((rows, cols), dtype=np.uint8)
        sb = np.empty((rows, cols // 16), dtype=np.uint8)
        g = np.zeros(1, dtype=np.float32)
        self._check("fm_get_nvfp4_weights", self.lib.fm_get_nvfp4_weights(self.h, layer, which, _ptr(codes),
                                                                           _ptr(sb), _ptr(g)))
        return codes, sb, np.float32(g[0])

    def quantize_act_e4m3(self, x_bits: np.ndarray, stream=None):
        """(codes [M, K] uint8, scales [M] fp32) of bf16 rows x_bits [M, K] by
        the W8A8 path's row-quantiser kernel."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        M, K = x.shape
        codes = np.empty((M, K), dtype=np.uint8)
        scales = np.empty(M, dtype=np.float32)
        self._check("fm_quantize_act_e4m3", self.lib.fm_quantize_act_e4m3(self.h, _ptr(x), M, K, _ptr(codes),
                                                                           _ptr(scales), _stream(stream)))
        return codes, scales

    def profile(self, batch: int, steps: int, iters: int, stream=None):
        """Mean (time-MLP ms, loop ms) over `iters` event-timed runs."""
        ms = np.zeros(2, dtype=np.float32)
        self._check("fm_profile_denoise", self.lib.fm_profile_denoise(self.h, batch, steps, iters, _ptr(ms),
                                                                       _stream(stream)))
        return float(ms[0]), float(ms[1])

    def profile_phases(self, steps: int, stream=None):
        """Timeline of one denoise (globaltimer ns, 0 where unused): compute
        marks [n_ctas, n_phases, 8], MMA marks [n_ctas, n_gemms, 2], chunk
        landed [n_ctas, n_chunks], chunk issued [n_ctas, n_chunks]."""
        n = ctypes.c_size_t(0)
        self._check("fm_profile_phases", self.lib.fm_profile_phases(self.h, steps, None, ctypes.byref(n), None))
        buf = np.zeros(n.value, dtype=np.uint64)
        self._check("fm_profile_phases", self.lib.fm_profile_phases(self.h, steps, _ptr(buf), ctypes.byref(n),
                                                                     _stream(stream)))
        L = self.shape.n_layers
        n_ph, n_g = steps * (2 + 5 * L), steps * 4 * L
        _, _, n_ctas = self.geometry()
        rows = buf.reshape(n_ctas, -1)
        n_ch = (rows.shape[1] - 16 * n_ph - 2 * n_g) // 2
        a, b = 16 * n_ph, 16 * n_ph + 2 * n_g
        return (rows[:, :a].reshape(n_ctas, n_ph, 16), rows[:, a:b].reshape(n_ctas, n_g, 2),
                rows[:, b:b + n_ch], rows[:, b + n_ch:b + 2 * n_ch])

    def sync(self, stream=None):
        self._check("fm_sync", self.lib.fm_sync(self.h, _stream(stream)))

    def test_stall(self, on: bool, spin_cycles: int = 0):
        """Test hook: make the loop kernel's QKV hand-off unreachable (see fm_test_stall)."""
        self._check("fm_test_stall", self.lib.fm_test_stall(self.h, 1 if on else 0, int(spin_cycles)))
