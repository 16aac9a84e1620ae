"""Python binding of libkie.so (argument marshalling only).

Every step of decode runs in the library's CUDA kernel; this module only
converts Python values to the C ABI of ``include/kie.h``. PyTorch is used for
device memory (output buffers) and for the current CUDA stream. There is no
fallback: if ``libkie.so`` is missing the import of ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkie.so")
# the same library compiled with KIE_TRACE (per-phase timestamps; measurement only)
LIB_TRACE_PATH = os.path.join(_HERE, "libkie_trace.so")

KIE_OK = 0
STATUS = {0: "KIE_OK", -1: "KIE_ERR_INVALID_ARG", -2: "KIE_ERR_STATE", -3: "KIE_ERR_CONTEXT_FULL",
          -4: "KIE_ERR_CUDA", -5: "KIE_ERR_TIMEOUT", -6: "KIE_ERR_DEVICE", -7: "KIE_ERR_OOM"}

EXPORTS = ["kie_create", "kie_load_weights", "kie_prefill", "kie_decode", "kie_decode_static",
           "kie_rewind", "kie_reset", "kie_destroy", "kie_last_error", "kie_position",
           "kie_pending", "kie_get_info", "kie_plan"]


class KieError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class kie_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
                 "n_experts", "top_k", "ffn_expert", "ffn_shared", "max_ctx")] + \
               [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


class kie_tensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("data", ctypes.c_void_p),
                ("shape", ctypes.c_int64 * 2), ("on_device", ctypes.c_int32)]


class kie_decode_opts(ctypes.Structure):
    _fields_ = [("forced_tokens", ctypes.c_void_p), ("logits_out", ctypes.c_void_p),
                ("margins_out", ctypes.c_void_p), ("timeout_ms", ctypes.c_uint32),
                ("fault_cta", ctypes.c_int32), ("fault_barrier", ctypes.c_int32),
                ("trace_out", ctypes.c_void_p), ("trace_cap", ctypes.c_int32),
                ("temperature", ctypes.c_float), ("top_k", ctypes.c_int32), ("top_p", ctypes.c_float),
                ("seed", ctypes.c_uint64)]


class kie_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("grid", "threads", "n_stages", "stage_bytes", "smem_bytes", "barriers_per_token")] + \
               [(n, ctypes.c_int64) for n in
                ("stream_bytes", "kv_bytes_per_pos", "resident_bytes", "launches")]


class kie_seg_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("K", "g", "nk", "kc")]


class kie_seg_range(ctypes.Structure):
    _fields_ = [("off", ctypes.c_int64), ("row0", ctypes.c_int32), ("nrows", ctypes.c_int32)]


class kie_plan_info(ctypes.Structure):
    _fields_ = [("slots", ctypes.c_int32), ("ranges_per_cta", ctypes.c_int32),
                ("tape_bytes", ctypes.c_int64), ("shapes", kie_seg_shape * 9)]


SEG_KINDS = ("qkv", "o", "gate_up", "down", "shared_gate_up", "expert_gate_up", "shared_down",
             "expert_down", "lm_head")

_libs = {}


def lib(trace: bool = False) -> ctypes.CDLL:
    """Load libkie.so (or, with ``trace``, libkie_trace.so), built in-tree;
    raises if it has not been built."""
    if trace in _libs:
        return _libs[trace]
    path = LIB_TRACE_PATH if trace else LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m transformer_decode_persistent_b200.build`")
    L = ctypes.CDLL(path)
    P, I, VP = ctypes.POINTER, ctypes.c_int, ctypes.c_void_p
    L.kie_create.argtypes = [P(kie_config), I, P(VP)]
    L.kie_load_weights.argtypes = [VP, P(kie_tensor), I, VP]
    L.kie_prefill.argtypes = [VP, P(ctypes.c_int32), I, VP]
    L.kie_decode.argtypes = [VP, I, VP, P(kie_decode_opts), VP]
    L.kie_decode_static.argtypes = [VP, I, VP, VP]
    L.kie_rewind.argtypes = [VP, ctypes.c_int32, ctypes.c_int32]
    L.kie_reset.argtypes = [VP]
    L.kie_destroy.argtypes = [VP]
    L.kie_last_error.argtypes = [VP]
    L.kie_last_error.restype = ctypes.c_char_p
    L.kie_position.argtypes = [VP]
    L.kie_position.restype = ctypes.c_int32
    L.kie_pending.argtypes = [VP]
    L.kie_pending.restype = ctypes.c_int32
    L.kie_get_info.argtypes = [VP, P(kie_info)]
    L.kie_plan.argtypes = [P(kie_config), ctypes.c_int32, ctypes.c_int32, P(kie_plan_info),
                           P(kie_seg_range), ctypes.c_int64]
    for f in ("kie_create", "kie_load_weights", "kie_prefill", "kie_decode", "kie_decode_static",
              "kie_rewind", "kie_reset", "kie_destroy", "kie_get_info", "kie_plan"):
        getattr(L, f).restype = ctypes.c_int
    _libs[trace] = L
    return L


def config_from(shape, max_ctx: int | None = None) -> kie_config:
    """kie_config from any object with the model-shape attributes."""
    g = lambda n, dflt=0: int(getattr(shape, n, dflt))
    return kie_config(n_layers=g("n_layers"), d_model=g("d_model"), n_heads=g("n_heads"),
                      n_kv_heads=g("n_kv_heads"), head_dim=g("head_dim"), ffn=g("ffn"),
                      vocab=g("vocab"), n_experts=g("n_experts"), top_k=g("top_k"),
                      ffn_expert=g("ffn_expert"), ffn_shared=g("ffn_shared"),
                      max_ctx=int(max_ctx if max_ctx is not None else shape.max_ctx),
                      rms_eps=float(shape.rms_eps), rope_theta=float(shape.rope_theta))


def plan(shape, grid: int, stage_bytes: int, max_ctx: int | None = None):
    """The weight-tape plan (kie_plan) for `grid` CTAs and ring stages of
    `stage_bytes`: (info dict with per-kind tile shapes, ranges as a structured
    numpy array [grid, ranges_per_cta] of (off, row0, nrows)). Host only."""
    L = lib()
    cfg = config_from(shape, max_ctx)
    info = kie_plan_info()
    st = L.kie_plan(ctypes.byref(cfg), int(grid), int(stage_bytes), ctypes.byref(info), None, 0)
    if st != KIE_OK:
        raise KieError(st, L.kie_last_error(None).decode())
    n = grid * info.ranges_per_cta
    buf = (kie_seg_range * n)()
    st = L.kie_plan(ctypes.byref(cfg), int(grid), int(stage_bytes), ctypes.byref(info), buf, n)
    if st != KIE_OK:
        raise KieError(st, L.kie_last_error(None).decode())
    dt = np.dtype([("off", np.int64), ("row0", np.int32), ("nrows", np.int32)])
    ranges = np.frombuffer(bytes(buf), dtype=dt).reshape(grid, info.ranges_per_cta)
    shapes = {k: dict(K=sh.K, g=sh.g, nk=sh.nk, kc=sh.kc) for k, sh in zip(SEG_KINDS, info.shapes)}
    return dict(slots=info.slots, ranges_per_cta=info.ranges_per_cta, tape_bytes=info.tape_bytes,
                shapes=shapes), ranges


def _check_out(out, n: int, device: int, need_cuda: bool = False):
    """Raise unless ``out`` can take n int32 tokens: a contiguous int32 tensor
    (CUDA on ``device``, or host) or a contiguous int32 numpy array."""
    import torch
    if isinstance(out, torch.Tensor):
        if out.dtype != torch.int32 or not out.is_contiguous() or out.numel() < n:
            raise ValueError(f"out must be a contiguous int32 tensor of >= {n} elements, got "
                             f"{out.dtype} {tuple(out.shape)}")
        if out.is_cuda and out.device.index != device:
            raise ValueError(f"out is on {out.device}, the engine on cuda:{device}")
        if need_cuda and not out.is_cuda:
            raise ValueError("out must be a CUDA tensor")
    else:
        if need_cuda:
            raise ValueError("out must be a CUDA tensor")
        a = out
        if not isinstance(a, np.ndarray) or a.dtype != np.int32 or not a.flags["C_CONTIGUOUS"] \
                or a.size < n:
            raise ValueError(f"out must be a contiguous int32 array of >= {n} elements")


def _stream_ptr(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


class Engine:
    """One batch-1 decode context on one GPU (a thin wrapper over kie_ctx)."""

    def __init__(self, shape, device: int = 0, max_ctx: int | None = None, trace_build: bool = False):
        """``trace_build`` loads libkie_trace.so, whose decode also writes one
        record of four phase timestamps per phase (see ``decode(trace=...)``)."""
        import torch
        self.trace_build = trace_build
        self.L = lib(trace_build)
        self.device = device
        self.cfg = config_from(shape, max_ctx)
        torch.cuda.init()
        with torch.cuda.device(device):
            h = ctypes.c_void_p()
            st = self.L.kie_create(ctypes.byref(self.cfg), device, ctypes.byref(h))
        if st != KIE_OK:
            raise KieError(st, self.L.kie_last_error(None).decode())
        self.h = h

    # -- helpers
    def _check(self, st: int):
        if st != KIE_OK:
            raise KieError(st, self.L.kie_last_error(self.h).decode())

    def close(self):
        if getattr(self, "h", None):
            self.L.kie_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    # -- API
    def load_weights(self, weights: dict, stream=None):
        """weights: name -> fp16 numpy array (host) or fp16 torch tensor (host or CUDA)."""
        import torch
        keep, arr = [], (kie_tensor * len(weights))()
        for i, (name, a) in enumerate(weights.items()):
            if isinstance(a, torch.Tensor):
                if a.dtype != torch.float16:
                    raise TypeError(f"{name}: expected float16, got {a.dtype}")
                a = a.contiguous()
                ptr, on_dev, shp = a.data_ptr(), int(a.is_cuda), tuple(a.shape)
            else:
                a = np.ascontiguousarray(a)
                if a.dtype != np.float16:
                    raise TypeError(f"{name}: expected float16, got {a.dtype}")
                ptr, on_dev, shp = a.ctypes.data, 0, a.shape
            keep.append(a)
            rows = int(shp[0])
            cols = int(shp[1]) if len(shp) > 1 else 1
            nb = name.encode()
            keep.append(nb)
            arr[i] = kie_tensor(nb, ptr, (ctypes.c_int64 * 2)(rows, cols), on_dev)
        with torch.cuda.device(self.device):
            self._check(self.L.kie_load_weights(self.h, arr, len(weights), _stream_ptr(stream)))

    def prefill(self, tokens, stream=None):
        import torch
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        with torch.cuda.device(self.device):
            self._check(self.L.kie_prefill(self.h, t.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                           len(t), _stream_ptr(stream)))

    def decode(self, n: int, forced=None, logits: bool = False, margins: bool = False,
               out=None, timeout_ms: int = 0, fault: tuple | None = None, trace=None,
               stream=None, temperature: float = 0.0, top_k: int = 0, top_p: float = 1.0,
               seed: int = 0):
        """Decode n tokens in one launch.

        Returns a dict with 'tokens' (numpy int32 [n], or the given ``out``),
        and 'logits' ([n, V] float32 CUDA tensor) / 'margins' ([n] float32 CUDA
        tensor) when requested. ``out`` may be a CUDA int32 tensor or a host
        (pinned) int32 tensor / numpy array. ``trace`` is a CUDA int64 tensor
        [grid, cap, 2] for the step barrier's arrival and release times, or,
        on a trace-build engine, [grid, cap, 4] with one record per phase
        (start, input ready, tiles done, epilogue done; records step * (5 L +
        2) + phase, the step barrier last). ``temperature`` > 0 samples in the
        kernel with ``top_k`` (1..64), ``top_p`` and the Philox ``seed``
        (see kie_decode_opts in include/kie.h); 0 is greedy.
        """
        import torch
        o = kie_decode_opts(fault_cta=-1, fault_barrier=-1, timeout_ms=int(timeout_ms),
                            temperature=float(temperature), top_k=int(top_k), top_p=float(top_p),
                            seed=int(seed) & 0xFFFFFFFFFFFFFFFF)
        keep = []
        if forced is not None:
            f = np.ascontiguousarray(np.asarray(forced, dtype=np.int32))
            keep.append(f)
            o.forced_tokens = f.ctypes.data
        res = {}
        dev = torch.device("cuda", self.device)
        if logits:
            lg = torch.empty((n, self.cfg.vocab), dtype=torch.float32, device=dev)
            o.logits_out = lg.data_ptr()
            res["logits"] = lg
        if margins:
            mg = torch.empty((n,), dtype=torch.float32, device=dev)
            o.margins_out = mg.data_ptr()
            res["margins"] = mg
        if fault is not None:
            o.fault_cta, o.fault_barrier = int(fault[0]), int(fault[1])
        if trace is not None:
            grid = self.info()["grid"]
            if (not isinstance(trace, torch.Tensor) or trace.dtype != torch.int64 or not trace.is_cuda
                    or trace.device.index != self.device or trace.dim() != 3
                    or trace.shape[0] != grid or trace.shape[2] != self.trace_words
                    or not trace.is_contiguous()):
                raise ValueError(f"trace must be a contiguous int64 CUDA tensor "
                                 f"[{grid}, cap, {self.trace_words}] on cuda:{self.device}")
            o.trace_out = trace.data_ptr()
            o.trace_cap = int(trace.shape[1])
        if out is None:
            out_arr = np.empty(n, dtype=np.int32)
            optr = out_arr.ctypes.data
            res["tokens"] = out_arr
        elif isinstance(out, torch.Tensor):
            _check_out(out, n, self.device)
            optr = out.data_ptr()
            res["tokens"] = out
        else:
            _check_out(out, n, self.device)
            optr = out.ctypes.data
            res["tokens"] = out
        with torch.cuda.device(self.device):
            self._check(self.L.kie_decode(self.h, int(n), ctypes.c_void_p(optr), ctypes.byref(o),
                                          _stream_ptr(stream)))
        return res

    def decode_static(self, n: int, out, stream=None):
        """kie_decode_static: n greedy tokens into ``out`` (a CUDA int32 tensor),
        with the kernel's scratch in the library's static device array."""
        import torch
        _check_out(out, n, self.device, need_cuda=True)
        with torch.cuda.device(self.device):
            self._check(self.L.kie_decode_static(self.h, int(n), ctypes.c_void_p(out.data_ptr()),
                                                 ctypes.c_void_p(_stream_ptr(stream))))
        return out

    def reset(self):
        self._check(self.L.kie_reset(self.h))

    def rewind(self, pos: int, pending: int):
        self._check(self.L.kie_rewind(self.h, int(pos), int(pending)))

    @property
    def trace_words(self) -> int:
        """Stamps per trace record: 4 in the trace build, 2 in the product."""
        return 4 if self.trace_build else 2

    @property
    def position(self) -> int:
        return int(self.L.kie_position(self.h))

    @property
    def pending(self) -> int:
        return int(self.L.kie_pending(self.h))

    def info(self) -> dict:
        inf = kie_info()
        self._check(self.L.kie_get_info(self.h, ctypes.byref(inf)))
        return {n: getattr(inf, n) for n, _ in kie_info._fields_}
