"""Python binding of the C-ABI in ``include/mono.h`` (ctypes).

Argument marshalling only: every step of the mixer runs in the CUDA kernels of
``libmono.so``.  There is no fallback: if the library is missing the import
fails.  PyTorch provides device memory and the stream; tensors are passed as
raw pointers after their shape, dtype, device and contiguity are checked.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmono.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m learned_product_hash_proj_b200.build` "
                      "(this package has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

MONO_F32, MONO_BF16 = 0, 1
MONO_FLAG_SIMPLE_KERNELS = 1
MONO_FLAG_REDIRECT = 2
STATUS = {0: "MONO_OK", 1: "MONO_ERR_INVALID", 2: "MONO_ERR_UNSUPPORTED", 3: "MONO_ERR_NULL",
          4: "MONO_ERR_WORKSPACE", 5: "MONO_ERR_CUDA", 6: "MONO_ERR_DEVICE", 7: "MONO_ERR_ALIGN", 8: "MONO_ERR_SCRATCH"}
REGIONS = {"kbar": 0, "addr": 1, "post_ids": 2, "post_addr": 3, "post_rank": 4, "overflow": 5, "Q": 6, "K": 7,
           "V": 8, "sel": 9, "O": 10, "walk_log": 11}
WALK_LOG_CAP = 4096
DEC_REGIONS = {"K": 0, "V": 1, "kbar": 2, "addr": 3, "count": 4, "head": 5, "tail": 6, "next": 7, "overflow": 8,
               "q": 9, "sel": 10, "o": 11}

EXPORTS = ("mono_plan", "mono_plan_destroy", "mono_workspace_region", "mono_project", "mono_route",
           "mono_route_summaries", "mono_route_lists", "mono_route_queries", "mono_attend",
           "mono_out_project", "mono_forward", "mono_stats", "mono_strerror", "mono_version", "mono_kernel_launches",
           "mono_route_static", "mono_route_static_capacity", "mono_decode_cache_bytes",
           "mono_decode_cache_region", "mono_decode_prefill", "mono_decode_project", "mono_decode_route",
           "mono_decode_attend", "mono_decode_step", "mono_backward_workspace_bytes", "mono_attend_backward",
           "mono_backward", "mono_out_project_scatter", "mono_stage_reduce", "mono_attend_pairs",
           "mono_attend_remote", "mono_attend_local")


class MonoError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = _lib.mono_strerror(status).decode()
        super().__init__(f"{what}: {STATUS.get(status, status)} ({msg})")


class _Config(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int) for k in ("B", "S", "W", "H", "d", "Bs", "L", "R", "E", "M", "C", "T", "cap")] + [
        ("rope_theta", ctypes.c_double), ("dtype", ctypes.c_int), ("flags", ctypes.c_int)]


class Stats(ctypes.Structure):
    _fields_ = [("overflow_total", ctypes.c_int64), ("overflow_max_bh", ctypes.c_int32),
                ("device_error", ctypes.c_int32), ("queries_lt_R", ctypes.c_int64),
                ("remote_selected", ctypes.c_int64), ("mean_remote", ctypes.c_double),
                ("forced_ignored", ctypes.c_int64), ("probe_walks", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


_P = ctypes.c_void_p
_lib.mono_plan.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_size_t)]
_lib.mono_plan_destroy.argtypes = [_P]
_lib.mono_plan_destroy.restype = None
_lib.mono_workspace_region.argtypes = [_P, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t),
                                       ctypes.POINTER(ctypes.c_size_t)]
_lib.mono_project.argtypes = [_P] * 10
_lib.mono_route.argtypes = [_P] * 8
_lib.mono_route_summaries.argtypes = [_P] * 5
_lib.mono_route_lists.argtypes = [_P] * 3
_lib.mono_route_queries.argtypes = [_P] * 7
_lib.mono_attend.argtypes = [_P] * 8
_lib.mono_out_project.argtypes = [_P] * 6
_lib.mono_forward.argtypes = [_P] * 11
_lib.mono_stats.argtypes = [_P, _P, _P, ctypes.POINTER(Stats)]
_lib.mono_strerror.argtypes = [ctypes.c_int]
_lib.mono_strerror.restype = ctypes.c_char_p
_lib.mono_version.argtypes = []
_lib.mono_route_static.argtypes = [_P] * 7
_lib.mono_route_static.restype = ctypes.c_int
_lib.mono_route_static_capacity.argtypes = []
_lib.mono_route_static_capacity.restype = ctypes.c_size_t
_lib.mono_decode_cache_bytes.argtypes = [_P, ctypes.POINTER(ctypes.c_size_t)]
_lib.mono_decode_cache_region.argtypes = [_P, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t),
                                          ctypes.POINTER(ctypes.c_size_t)]
_lib.mono_decode_prefill.argtypes = [_P, ctypes.c_int, _P, _P, _P]
_lib.mono_decode_project.argtypes = [_P, ctypes.c_int] + [_P] * 6
_lib.mono_decode_route.argtypes = [_P, ctypes.c_int] + [_P] * 4
_lib.mono_decode_attend.argtypes = [_P, ctypes.c_int, _P, _P]
_lib.mono_decode_step.argtypes = [_P, ctypes.c_int] + [_P] * 10
_lib.mono_backward_workspace_bytes.argtypes = [_P, ctypes.POINTER(ctypes.c_size_t)]
_lib.mono_attend_backward.argtypes = [_P] * 11
_lib.mono_backward.argtypes = [_P] * 16
_lib.mono_out_project_scatter.argtypes = [_P, _P, _P, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int,
                                          _P, _P]
_lib.mono_stage_reduce.argtypes = [_P, _P, ctypes.c_int, _P, _P]
_lib.mono_attend_pairs.argtypes = [_P] * 4
_lib.mono_attend_remote.argtypes = [_P] * 6
_lib.mono_attend_local.argtypes = [_P] * 8
_lib.mono_kernel_launches.argtypes = []
_lib.mono_kernel_launches.restype = ctypes.c_ulonglong
for _f in ("mono_plan", "mono_workspace_region", "mono_project", "mono_route", "mono_route_summaries",
           "mono_route_lists", "mono_route_queries", "mono_attend", "mono_out_project",
           "mono_forward", "mono_stats", "mono_version", "mono_decode_cache_bytes", "mono_decode_cache_region",
           "mono_decode_prefill", "mono_decode_project", "mono_decode_route", "mono_decode_attend",
           "mono_decode_step", "mono_backward_workspace_bytes", "mono_attend_backward", "mono_backward",
           "mono_out_project_scatter", "mono_stage_reduce", "mono_attend_pairs", "mono_attend_remote",
           "mono_attend_local"):
    getattr(_lib, _f).restype = ctypes.c_int


def lib() -> ctypes.CDLL:
    return _lib


def _check(st: int, what: str):
    if st != 0:
        raise MonoError(st, what)


def _torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


class Plan:
    """An immutable plan for one shape/method configuration.

    `cfg` is any object with the fields B S W H d Bs L R E M C T cap theta
    dtype ("f32" | "bf16") -- e.g. ``synth.config("scale32k")``.
    """

    def __init__(self, cfg, flags: int = 0):
        self.cfg = cfg
        self.flags = flags
        self.dtype = _torch_dtype(cfg.dtype)
        c = _Config(*(int(getattr(cfg, k)) for k in ("B", "S", "W", "H", "d", "Bs", "L", "R", "E", "M", "C", "T",
                                                        "cap")),
                    float(getattr(cfg, "theta", 10000.0)), MONO_BF16 if cfg.dtype == "bf16" else MONO_F32, int(flags))
        h = _P()
        ws = ctypes.c_size_t()
        _check(_lib.mono_plan(ctypes.byref(c), ctypes.byref(h), ctypes.byref(ws)), "mono_plan")
        self._h = h
        self._destroy = _lib.mono_plan_destroy
        self.workspace_bytes = int(ws.value)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def workspace(self, device="cuda") -> torch.Tensor:
        """A caller-owned workspace tensor of the size this plan needs."""
        return torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8, device=device)

    def region(self, ws: torch.Tensor, name: str) -> torch.Tensor:
        """A typed view of a workspace region (see mono_ws_region)."""
        off, nbytes = ctypes.c_size_t(), ctypes.c_size_t()
        _check(_lib.mono_workspace_region(self._h, REGIONS[name], ctypes.byref(off), ctypes.byref(nbytes)),
               "mono_workspace_region")
        c = self.cfg
        nb = c.S // c.Bs
        shapes = {"kbar": ((c.B, c.H, nb, c.d), torch.float32), "addr": ((c.B, c.H, nb), torch.int32),
                  "post_ids": ((c.B, c.H, nb), torch.int32), "post_addr": ((c.B, c.H, nb), torch.int32),
                  "post_rank": ((c.B, c.H, nb), torch.int32), "overflow": ((c.B, c.H), torch.int32),
                  "Q": ((c.B, c.H, c.S, c.d), self.dtype), "K": ((c.B, c.H, c.S, c.d), self.dtype),
                  "V": ((c.B, c.H, c.S, c.d), self.dtype), "sel": ((c.B, c.H, c.S, c.R), torch.int32),
                  "O": ((c.B, c.S, c.H * c.d), self.dtype), "walk_log": ((WALK_LOG_CAP,), torch.int32)}
        shape, dt = shapes[name]
        raw = ws[off.value:off.value + nbytes.value]
        return raw.view(dt).view(shape)


def _ptr(t, what, shape=None, dtype=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{what} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def project(plan: Plan, x, Wq, Wk, Wv, Q, K, V, ws, stream=None):
    c, dt = plan.cfg, plan.dtype
    hd = c.H * c.d
    qkv = (c.B, c.H, c.S, c.d)
    _check(_lib.mono_project(plan.handle, _ptr(x, "x", (c.B, c.S, c.W), dt), _ptr(Wq, "Wq", (hd, c.W), dt),
                             _ptr(Wk, "Wk", (hd, c.W), dt), _ptr(Wv, "Wv", (hd, c.W), dt), _ptr(Q, "Q", qkv, dt),
                             _ptr(K, "K", qkv, dt), _ptr(V, "V", qkv, dt), _ptr(ws, "workspace"), _stream(stream)),
           "mono_project")


def route(plan: Plan, Q, K, codebooks, sel, ws, forced=None, stream=None):
    c, dt = plan.cfg, plan.dtype
    qkv = (c.B, c.H, c.S, c.d)
    _check(_lib.mono_route(plan.handle, _ptr(Q, "Q", qkv, dt), _ptr(K, "K", qkv, dt),
                           _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                           _ptr(forced, "forced", (c.B, c.H, c.S), torch.int32, optional=True),
                           _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32), _ptr(ws, "workspace"),
                           _stream(stream)), "mono_route")


def route_summaries(plan: Plan, K, codebooks, ws, stream=None):
    c, dt = plan.cfg, plan.dtype
    _check(_lib.mono_route_summaries(plan.handle, _ptr(K, "K", (c.B, c.H, c.S, c.d), dt),
                                     _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                                     _ptr(ws, "workspace"), _stream(stream)), "mono_route_summaries")


def route_lists(plan: Plan, ws, stream=None):
    _check(_lib.mono_route_lists(plan.handle, _ptr(ws, "workspace"), _stream(stream)), "mono_route_lists")


def route_queries(plan: Plan, Q, codebooks, sel, ws, forced=None, stream=None):
    c, dt = plan.cfg, plan.dtype
    _check(_lib.mono_route_queries(plan.handle, _ptr(Q, "Q", (c.B, c.H, c.S, c.d), dt),
                                   _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                                   _ptr(forced, "forced", (c.B, c.H, c.S), torch.int32, optional=True),
                                   _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32), _ptr(ws, "workspace"),
                                   _stream(stream)), "mono_route_queries")


def route_static(plan: Plan, Q, K, codebooks, sel, forced=None, stream=None):
    """mono_route without a workspace, for callers that cannot allocate device memory.

    The routing tables live in a fixed array owned by the library (see
    mono_route_static in include/mono.h); calls that overlap on the GPU race.
    """
    c, dt = plan.cfg, plan.dtype
    qkv = (c.B, c.H, c.S, c.d)
    _check(_lib.mono_route_static(plan.handle, _ptr(Q, "Q", qkv, dt), _ptr(K, "K", qkv, dt),
                                  _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                                  _ptr(forced, "forced", (c.B, c.H, c.S), torch.int32, optional=True),
                                  _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32), _stream(stream)),
           "mono_route_static")


def attend(plan: Plan, Q, K, V, sel, O, ws, stream=None):
    c, dt = plan.cfg, plan.dtype
    qkv = (c.B, c.H, c.S, c.d)
    _check(_lib.mono_attend(plan.handle, _ptr(Q, "Q", qkv, dt), _ptr(K, "K", qkv, dt), _ptr(V, "V", qkv, dt),
                            _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32),
                            _ptr(O, "O", (c.B, c.S, c.H * c.d), dt), _ptr(ws, "workspace"), _stream(stream)),
           "mono_attend")


def attend_pairs(plan: Plan, sel, ws, stream=None):
    c = plan.cfg
    _check(_lib.mono_attend_pairs(plan.handle, _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32,
                                                    optional=c.R == 0),
                                  _ptr(ws, "workspace"), _stream(stream)), "mono_attend_pairs")


def attend_remote(plan: Plan, Q, K, V, ws, stream=None):
    c, dt = plan.cfg, plan.dtype
    qkv = (c.B, c.H, c.S, c.d)
    _check(_lib.mono_attend_remote(plan.handle, _ptr(Q, "Q", qkv, dt), _ptr(K, "K", qkv, dt), _ptr(V, "V", qkv, dt),
                                   _ptr(ws, "workspace"), _stream(stream)), "mono_attend_remote")


def attend_local(plan: Plan, Q, K, V, sel, O, ws, stream=None):
    c, dt = plan.cfg, plan.dtype
    qkv = (c.B, c.H, c.S, c.d)
    _check(_lib.mono_attend_local(plan.handle, _ptr(Q, "Q", qkv, dt), _ptr(K, "K", qkv, dt), _ptr(V, "V", qkv, dt),
                                  _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32, optional=c.R == 0),
                                  _ptr(O, "O", (c.B, c.S, c.H * c.d), dt), _ptr(ws, "workspace"), _stream(stream)),
           "mono_attend_local")


def out_project(plan: Plan, O, Wo, delta, ws, stream=None):
    c, dt = plan.cfg, plan.dtype
    _check(_lib.mono_out_project(plan.handle, _ptr(O, "O", (c.B, c.S, c.H * c.d), dt),
                                 _ptr(Wo, "Wo", (c.W, c.H * c.d), dt), _ptr(delta, "delta", (c.B, c.S, c.W), dt),
                                 _ptr(ws, "workspace"), _stream(stream)), "mono_out_project")


def out_project_scatter(plan: Plan, O, Wo, stages, rank: int, ws, stream=None):
    """The head shard's output projection into the owners' staging buffers (mono_out_project_scatter).
    `stages`: one entry per rank c -- rank c's fp32 staging buffer [N, B*S/N, W], as a CUDA tensor of this
    device or as a raw device address (int) of peer-accessible memory."""
    c, dt = plan.cfg, plan.dtype
    n = len(stages)
    ptrs = (ctypes.c_void_p * n)()
    for r, st in enumerate(stages):
        if isinstance(st, torch.Tensor):
            ptrs[r] = _ptr(st, f"stage[{r}]", (n, c.B * c.S // n, c.W), torch.float32).value
        else:
            ptrs[r] = int(st)
    _check(_lib.mono_out_project_scatter(plan.handle, _ptr(O, "O", (c.B, c.S, c.H * c.d), dt),
                                         _ptr(Wo, "Wo", (c.W, c.H * c.d), dt), ptrs, ctypes.c_int(n),
                                         ctypes.c_int(rank), _ptr(ws, "workspace"), _stream(stream)),
           "mono_out_project_scatter")


def stage_reduce(plan: Plan, stage, nranks: int, delta_chunk, stream=None):
    """The owner's fixed-order fp32 sum of its staged partials, rounded once (mono_stage_reduce)."""
    c, dt = plan.cfg, plan.dtype
    rows = c.B * c.S // nranks
    _check(_lib.mono_stage_reduce(plan.handle, _ptr(stage, "stage", (nranks, rows, c.W), torch.float32),
                                  ctypes.c_int(nranks), _ptr(delta_chunk, "delta_chunk", (rows, c.W), dt),
                                  _stream(stream)), "mono_stage_reduce")


def forward(plan: Plan, x, Wq, Wk, Wv, Wo, codebooks, delta, ws, forced=None, stream=None):
    c, dt = plan.cfg, plan.dtype
    hd = c.H * c.d
    _check(_lib.mono_forward(plan.handle, _ptr(x, "x", (c.B, c.S, c.W), dt), _ptr(Wq, "Wq", (hd, c.W), dt),
                             _ptr(Wk, "Wk", (hd, c.W), dt), _ptr(Wv, "Wv", (hd, c.W), dt),
                             _ptr(Wo, "Wo", (c.W, hd), dt),
                             _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                             _ptr(forced, "forced", (c.B, c.H, c.S), torch.int32, optional=True),
                             _ptr(delta, "delta", (c.B, c.S, c.W), dt), _ptr(ws, "workspace"), _stream(stream)),
           "mono_forward")


def stats(plan: Plan, ws, stream=None, check: bool = True) -> dict:
    st = Stats()
    rc = _lib.mono_stats(plan.handle, _ptr(ws, "workspace"), _stream(stream), ctypes.byref(st))
    if check:
        _check(rc, "mono_stats")
    d = st.as_dict()
    d["status"] = rc
    return d


# ---------------------------------------------------------------------------
# decode: one new token per sequence against a caller-owned cache
# ---------------------------------------------------------------------------
def decode_cache(plan: Plan, device="cuda") -> torch.Tensor:
    """A caller-owned decode cache (uint8) of the size mono_decode_cache_bytes gives."""
    n = ctypes.c_size_t()
    _check(_lib.mono_decode_cache_bytes(plan.handle, ctypes.byref(n)), "mono_decode_cache_bytes")
    return torch.zeros(max(int(n.value), 256), dtype=torch.uint8, device=device)


def decode_region(plan: Plan, cache: torch.Tensor, name: str) -> torch.Tensor:
    """A typed view of a decode-cache region (see mono_dec_region)."""
    off, nbytes = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.mono_decode_cache_region(plan.handle, DEC_REGIONS[name], ctypes.byref(off), ctypes.byref(nbytes)),
           "mono_decode_cache_region")
    c = plan.cfg
    nb, A = c.S // c.Bs, c.C ** c.M
    shapes = {"K": ((c.B, c.H, c.S, c.d), plan.dtype), "V": ((c.B, c.H, c.S, c.d), plan.dtype),
              "kbar": ((c.B, c.H, nb, c.d), torch.float32), "addr": ((c.B, c.H, nb), torch.int32),
              "count": ((c.B, c.H, A), torch.int32), "head": ((c.B, c.H, A), torch.int32),
              "tail": ((c.B, c.H, A), torch.int32), "next": ((c.B, c.H, nb), torch.int32),
              "overflow": ((c.B, c.H), torch.int32), "q": ((c.B, c.H, c.d), plan.dtype),
              "sel": ((c.B, c.H, max(c.R, 1)), torch.int32), "o": ((c.B, c.H * c.d), plan.dtype)}
    shape, dt = shapes[name]
    raw = cache[off.value:off.value + nbytes.value]
    return raw.view(dt).view(shape)


def decode_prefill(plan: Plan, t0: int, codebooks, cache, stream=None):
    c = plan.cfg
    _check(_lib.mono_decode_prefill(plan.handle, int(t0),
                                    _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                                    _ptr(cache, "cache"), _stream(stream)), "mono_decode_prefill")


def decode_project(plan: Plan, t: int, x_t, Wq, Wk, Wv, cache, stream=None):
    c, dt = plan.cfg, plan.dtype
    hd = c.H * c.d
    _check(_lib.mono_decode_project(plan.handle, int(t), _ptr(x_t, "x_t", (c.B, c.W), dt),
                                    _ptr(Wq, "Wq", (hd, c.W), dt), _ptr(Wk, "Wk", (hd, c.W), dt),
                                    _ptr(Wv, "Wv", (hd, c.W), dt), _ptr(cache, "cache"), _stream(stream)),
           "mono_decode_project")


def decode_route(plan: Plan, t: int, codebooks, cache, forced_t=None, stream=None):
    c = plan.cfg
    _check(_lib.mono_decode_route(plan.handle, int(t),
                                  _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                                  _ptr(forced_t, "forced_t", (c.B, c.H), torch.int32, optional=True),
                                  _ptr(cache, "cache"), _stream(stream)), "mono_decode_route")


def decode_attend(plan: Plan, t: int, cache, stream=None):
    _check(_lib.mono_decode_attend(plan.handle, int(t), _ptr(cache, "cache"), _stream(stream)), "mono_decode_attend")


def decode_step(plan: Plan, t: int, x_t, Wq, Wk, Wv, Wo, codebooks, delta_t, cache, forced_t=None, stream=None):
    c, dt = plan.cfg, plan.dtype
    hd = c.H * c.d
    _check(_lib.mono_decode_step(plan.handle, int(t), _ptr(x_t, "x_t", (c.B, c.W), dt),
                                 _ptr(Wq, "Wq", (hd, c.W), dt), _ptr(Wk, "Wk", (hd, c.W), dt),
                                 _ptr(Wv, "Wv", (hd, c.W), dt), _ptr(Wo, "Wo", (c.W, hd), dt),
                                 _ptr(codebooks, "codebooks", (c.H, c.M, c.C, c.d // c.M), torch.float32),
                                 _ptr(forced_t, "forced_t", (c.B, c.H), torch.int32, optional=True),
                                 _ptr(delta_t, "delta_t", (c.B, c.W), dt), _ptr(cache, "cache"), _stream(stream)),
           "mono_decode_step")


# ---------------------------------------------------------------------------
# backward pass for a fixed selection
# ---------------------------------------------------------------------------
def backward_workspace(plan: Plan, device="cuda") -> torch.Tensor:
    """A caller-owned backward workspace of the size mono_backward_workspace_bytes gives."""
    n = ctypes.c_size_t()
    _check(_lib.mono_backward_workspace_bytes(plan.handle, ctypes.byref(n)), "mono_backward_workspace_bytes")
    return torch.empty(max(int(n.value), 256), dtype=torch.uint8, device=device)


def attend_backward(plan: Plan, Q, K, V, sel, dO, dQ, dK, dV, bws, stream=None):
    c, dt = plan.cfg, plan.dtype
    qkv = (c.B, c.H, c.S, c.d)
    f32 = torch.float32
    _check(_lib.mono_attend_backward(plan.handle, _ptr(Q, "Q", qkv, dt), _ptr(K, "K", qkv, dt), _ptr(V, "V", qkv, dt),
                                     _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32),
                                     _ptr(dO, "dO", (c.B, c.S, c.H * c.d), f32), _ptr(dQ, "dQ", qkv, f32),
                                     _ptr(dK, "dK", qkv, f32), _ptr(dV, "dV", qkv, f32),
                                     _ptr(bws, "bwd_workspace"), _stream(stream)), "mono_attend_backward")


def backward(plan: Plan, x, Wq, Wk, Wv, Wo, sel, ddelta, dx, dWq, dWk, dWv, dWo, ws, bws, stream=None):
    c, dt = plan.cfg, plan.dtype
    hd = c.H * c.d
    f32 = torch.float32
    _check(_lib.mono_backward(plan.handle, _ptr(x, "x", (c.B, c.S, c.W), dt), _ptr(Wq, "Wq", (hd, c.W), dt),
                              _ptr(Wk, "Wk", (hd, c.W), dt), _ptr(Wv, "Wv", (hd, c.W), dt),
                              _ptr(Wo, "Wo", (c.W, hd), dt), _ptr(sel, "sel", (c.B, c.H, c.S, c.R), torch.int32),
                              _ptr(ddelta, "ddelta", (c.B, c.S, c.W), dt), _ptr(dx, "dx", (c.B, c.S, c.W), f32),
                              _ptr(dWq, "dWq", (hd, c.W), f32), _ptr(dWk, "dWk", (hd, c.W), f32),
                              _ptr(dWv, "dWv", (hd, c.W), f32), _ptr(dWo, "dWo", (c.W, hd), f32),
                              _ptr(ws, "workspace"), _ptr(bws, "bwd_workspace"), _stream(stream)), "mono_backward")


def version() -> int:
    return _lib.mono_version()


def kernel_launches() -> int:
    """Kernels launched by libmono.so in this process so far."""
    return int(_lib.mono_kernel_launches())
