"""Python binding of the B200 MoE-layer library (include/moe.h).

Argument marshalling only: every function here forwards to the C ABI entry
point of the same name in libmoe_b200.so, passing torch tensors' device
addresses.  There is no fallback: if the library is missing or a call fails,
an exception is raised.  PyTorch supplies device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE = -5

MOE_W_BF16 = 0
MOE_W_FP8_E4M3_B128 = 1

MOE_DEV_WAIT_TIMEOUT_GATE_UP = 0x1
MOE_DEV_WAIT_TIMEOUT_DOWN = 0x2
MOE_DEV_BAD_EXPERT_ID = 0x4
MOE_DEV_WAIT_TIMEOUT_ROUTER = 0x8
MOE_DEV_WAIT_TIMEOUT_SEND = 0x10

MOE_NUM_STAGES = 7
STAGE_NAMES = ("router", "topk", "permute", "gather", "gate_up_gemm", "down_gemm", "combine")

EXPORTED = ("moe_plan_create", "moe_plan_destroy", "moe_plan_set_wait_limit", "moe_forward",
            "moe_forward_scatter", "moe_forward_scatter_experts", "moe_reduce_partials",
            "moe_route_from_logits", "moe_route_from_logits_noalloc", "moe_check_device_status",
            "moe_get_workspace_views", "moe_status_string", "moe_last_cuda_error_string",
            "moe_pipeline_slot_bytes", "moe_pipeline_create", "moe_pipeline_submit",
            "moe_pipeline_synchronize", "moe_pipeline_streams", "moe_pipeline_destroy",
            "moe_router_split_bytes", "moe_split_router_weights", "moe_forward_scatter_pairs",
            "moe_reduce_pairs")
MAX_TP_RANKS = 8

MOE_STATIC_SCRATCH_BYTES = 4 << 20

_c_int = ctypes.c_int
_vp = ctypes.c_void_p


class moe_config(ctypes.Structure):
    _fields_ = [("max_tokens", _c_int), ("hidden", _c_int), ("num_experts", _c_int),
                ("top_k_max", _c_int), ("inter", _c_int), ("num_shared", _c_int),
                ("shared_inter", _c_int), ("renormalize", _c_int), ("wtype", _c_int)]


class moe_weights(ctypes.Structure):
    _fields_ = [("router_w", _vp), ("router_b", _vp), ("w_gate_up", _vp), ("w_down", _vp),
                ("s_gate_up", _vp), ("s_down", _vp), ("ws_gate_up", _vp), ("ws_down", _vp),
                ("ss_gate_up", _vp), ("ss_down", _vp), ("router_split", _vp)]


class moe_debug(ctypes.Structure):
    _fields_ = [("logits", _vp), ("topk_ids", _vp), ("topk_w", _vp), ("perm", _vp),
                ("offsets", _vp), ("events", _vp * (MOE_NUM_STAGES + 1))]


class moe_workspace_views(ctypes.Structure):
    _fields_ = [("row_token", _vp), ("x_perm", _vp), ("h", _vp), ("y", _vp),
                ("group_offsets", _vp), ("h_stride", _c_int), ("x_scale", _vp),
                ("h_scale", _vp)]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = f": {moe_last_cuda_error_string()}" if status == MOE_ERR_CUDA else ""
        super().__init__(f"{where}: {moe_status_string(status)} ({status}){detail}")


_lib = None


def load():
    """Loads libmoe_b200.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run mixture_experts_fp32_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    L.moe_plan_create.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(_vp),
                                  ctypes.POINTER(ctypes.c_size_t)]
    L.moe_plan_create.restype = _c_int
    L.moe_plan_destroy.argtypes = [_vp]
    L.moe_plan_destroy.restype = None
    L.moe_plan_set_wait_limit.argtypes = [_vp, ctypes.c_uint64]
    L.moe_plan_set_wait_limit.restype = _c_int
    L.moe_forward.argtypes = [_vp, ctypes.POINTER(moe_weights), _vp, _vp, _c_int, _c_int, _vp, _vp,
                              ctypes.c_size_t, _vp, ctypes.POINTER(moe_debug)]
    L.moe_forward.restype = _c_int
    L.moe_forward_scatter.argtypes = [_vp, ctypes.POINTER(moe_weights), _vp, _vp, _c_int, _c_int,
                                      ctypes.POINTER(_vp), _c_int, _c_int, _c_int, _vp,
                                      ctypes.c_size_t, _vp, ctypes.POINTER(moe_debug)]
    L.moe_forward_scatter.restype = _c_int
    L.moe_forward_scatter_experts.argtypes = [_vp, ctypes.POINTER(moe_weights), _vp, _vp, _c_int,
                                              _c_int, ctypes.POINTER(_vp), _c_int, _c_int, _c_int,
                                              _c_int, _c_int, _vp, ctypes.c_size_t, _vp,
                                              ctypes.POINTER(moe_debug)]
    L.moe_forward_scatter_experts.restype = _c_int
    L.moe_reduce_partials.argtypes = [_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]
    L.moe_reduce_partials.restype = _c_int
    L.moe_route_from_logits.argtypes = [_vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp,
                                        ctypes.c_size_t, _vp]
    L.moe_route_from_logits.restype = _c_int
    L.moe_route_from_logits_noalloc.argtypes = [_vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _vp,
                                                _vp, _vp]
    L.moe_route_from_logits_noalloc.restype = _c_int
    L.moe_check_device_status.argtypes = [_vp, _vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
    L.moe_check_device_status.restype = _c_int
    L.moe_get_workspace_views.argtypes = [_vp, _vp, ctypes.POINTER(moe_workspace_views)]
    L.moe_get_workspace_views.restype = _c_int
    L.moe_status_string.argtypes = [_c_int]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_last_cuda_error_string.argtypes = []
    L.moe_last_cuda_error_string.restype = ctypes.c_char_p
    L.moe_pipeline_slot_bytes.argtypes = [_vp, _c_int, _c_int, ctypes.POINTER(ctypes.c_size_t)]
    L.moe_pipeline_slot_bytes.restype = _c_int
    L.moe_pipeline_create.argtypes = [_vp, ctypes.POINTER(moe_weights), _c_int, _c_int, _c_int,
                                      _c_int, _vp, ctypes.c_size_t, _vp, ctypes.c_size_t,
                                      ctypes.POINTER(_vp)]
    L.moe_pipeline_create.restype = _c_int
    L.moe_pipeline_submit.argtypes = [_vp, _vp, _vp, _vp]
    L.moe_pipeline_submit.restype = _c_int
    L.moe_pipeline_synchronize.argtypes = [_vp]
    L.moe_pipeline_synchronize.restype = _c_int
    L.moe_pipeline_streams.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                       ctypes.POINTER(_vp)]
    L.moe_pipeline_streams.restype = _c_int
    L.moe_forward_scatter_pairs.argtypes = [_vp, ctypes.POINTER(moe_weights), _vp, _vp, _c_int,
                                            _c_int, _vp, _c_int, _c_int, _c_int, _c_int,
                                            _c_int, _c_int, _vp, ctypes.c_size_t, _vp, _vp]
    L.moe_forward_scatter_pairs.restype = _c_int
    L.moe_reduce_pairs.argtypes = [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp]
    L.moe_reduce_pairs.restype = _c_int
    L.moe_router_split_bytes.argtypes = [_vp]
    L.moe_router_split_bytes.restype = ctypes.c_size_t
    L.moe_split_router_weights.argtypes = [_vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.moe_split_router_weights.restype = _c_int
    L.moe_pipeline_destroy.argtypes = [_vp]
    L.moe_pipeline_destroy.restype = None
    _lib = L
    return L


# element types accepted for each kind of tensor argument (torch dtype names)
_F32 = ("float32",)
_I32 = ("int32",)
_BF16 = ("bfloat16",)
_MASK = ("uint8", "bool")
_WEIGHT = ("bfloat16", "uint8", "float8_e4m3fn")


def _addr(t, name: str = "argument", dtypes=None) -> int | None:
    """Address of a tensor argument, or an int taken as a raw address, or None.

    A tensor must be a contiguous CUDA tensor (of one of ``dtypes`` when given):
    the kernels read and write it as a dense row-major array in device memory, so a
    host tensor, a strided view or a wrong element type is refused here, before
    anything is enqueued, instead of being read out of bounds on the device."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"{name}: a CUDA tensor is required, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: a contiguous tensor is required")
    if dtypes is not None and str(t.dtype).rsplit(".", 1)[-1] not in dtypes:
        raise ValueError(f"{name}: element type {t.dtype} is not one of {', '.join(dtypes)}")
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def moe_status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def moe_last_cuda_error_string() -> str:
    return load().moe_last_cuda_error_string().decode()


def moe_plan_create(cfg: moe_config):
    """Returns (plan handle, workspace bytes)."""
    plan = _vp()
    ws = ctypes.c_size_t()
    _check(load().moe_plan_create(ctypes.byref(cfg), ctypes.byref(plan), ctypes.byref(ws)),
           "moe_plan_create")
    return plan.value, ws.value


def moe_plan_destroy(plan) -> None:
    load().moe_plan_destroy(plan)


def moe_plan_set_wait_limit(plan, limit_ns: int) -> None:
    _check(load().moe_plan_set_wait_limit(plan, limit_ns), "moe_plan_set_wait_limit")


def make_weights(router_w, router_b=None, w_gate_up=None, w_down=None, s_gate_up=None,
                 s_down=None, ws_gate_up=None, ws_down=None, ss_gate_up=None,
                 ss_down=None, router_split=None) -> moe_weights:
    return moe_weights(_addr(router_w, "router_w", _F32), _addr(router_b, "router_b", _F32),
                       _addr(w_gate_up, "w_gate_up", _WEIGHT), _addr(w_down, "w_down", _WEIGHT),
                       _addr(s_gate_up, "s_gate_up", _F32), _addr(s_down, "s_down", _F32),
                       _addr(ws_gate_up, "ws_gate_up", _WEIGHT), _addr(ws_down, "ws_down", _WEIGHT),
                       _addr(ss_gate_up, "ss_gate_up", _F32), _addr(ss_down, "ss_down", _F32),
                       _addr(router_split, "router_split", _BF16))


def moe_router_split_bytes(plan) -> int:
    return int(load().moe_router_split_bytes(plan))


def moe_split_router_weights(plan, router_w, split, split_bytes: int, stream=None) -> None:
    _check(load().moe_split_router_weights(plan, _addr(router_w, "router_w", _F32),
                                           _addr(split, "split", _BF16), split_bytes,
                                           _stream(stream)), "moe_split_router_weights")


def make_debug(logits=None, topk_ids=None, topk_w=None, perm=None, offsets=None,
               events=None) -> moe_debug:
    d = moe_debug(_addr(logits, "logits", _F32), _addr(topk_ids, "topk_ids", _I32),
                  _addr(topk_w, "topk_w", _F32), _addr(perm, "perm", _I32),
                  _addr(offsets, "offsets", _I32))
    if events is not None:
        for i, ev in enumerate(events):
            d.events[i] = None if ev is None else ev.cuda_event
    return d


def moe_forward(plan, weights: moe_weights, hidden, valid, T: int, k: int, out, workspace,
                ws_bytes: int, stream=None, dbg: moe_debug | None = None) -> None:
    st = load().moe_forward(plan, ctypes.byref(weights), _addr(hidden, "hidden", _BF16),
                            _addr(valid, "valid", _MASK), T, k, _addr(out, "out", _BF16),
                            _addr(workspace, "workspace"), ws_bytes, _stream(stream),
                            None if dbg is None else ctypes.byref(dbg))
    _check(st, "moe_forward")


def moe_forward_scatter(plan, weights: moe_weights, hidden, valid, T: int, k: int, dst,
                        rows_per_rank: int, slot: int, workspace, ws_bytes: int, stream=None,
                        dbg: moe_debug | None = None) -> None:
    """dst: a sequence of device addresses (or tensors) of the owners' receive slabs."""
    arr = (_vp * len(dst))(*[_addr(d, "dst", _F32) for d in dst])
    st = load().moe_forward_scatter(plan, ctypes.byref(weights), _addr(hidden, "hidden", _BF16),
                                    _addr(valid, "valid", _MASK), T, k,
                                    arr, len(dst), rows_per_rank, slot, _addr(workspace, "workspace"),
                                    ws_bytes, _stream(stream),
                                    None if dbg is None else ctypes.byref(dbg))
    _check(st, "moe_forward_scatter")


def moe_forward_scatter_experts(plan, weights: moe_weights, hidden, valid, T: int, k: int, dst,
                                rows_per_rank: int, slot: int, expert_begin: int, expert_end: int,
                                workspace, ws_bytes: int, stream=None,
                                dbg: moe_debug | None = None) -> None:
    arr = (_vp * len(dst))(*[_addr(d, "dst", _F32) for d in dst])
    st = load().moe_forward_scatter_experts(plan, ctypes.byref(weights),
                                            _addr(hidden, "hidden", _BF16),
                                            _addr(valid, "valid", _MASK), T, k, arr, len(dst),
                                            rows_per_rank, slot, expert_begin, expert_end,
                                            _addr(workspace, "workspace"),
                                            ws_bytes, _stream(stream),
                                            None if dbg is None else ctypes.byref(dbg))
    _check(st, "moe_forward_scatter_experts")


def moe_forward_scatter_pairs(plan, weights: moe_weights, hidden, valid, T: int, k: int, dst,
                              rows_per_rank: int, shared_slot: int, expert_begin: int,
                              expert_end: int, send_ctas: int, workspace, ws_bytes: int,
                              stream=None, dbg: moe_debug | None = None) -> None:
    """dst: the owners' per-pair receive slabs (device addresses or tensors)."""
    arr = (_vp * len(dst))(*[_addr(d, "dst", _F32) for d in dst])
    st = load().moe_forward_scatter_pairs(plan, ctypes.byref(weights),
                                          _addr(hidden, "hidden", _BF16),
                                          _addr(valid, "valid", _MASK), T, k, arr, len(dst),
                                          rows_per_rank, shared_slot, expert_begin, expert_end,
                                          send_ctas, _addr(workspace, "workspace"), ws_bytes,
                                          _stream(stream),
                                          None if dbg is None else ctypes.byref(dbg))
    _check(st, "moe_forward_scatter_pairs")


def moe_reduce_pairs(slab, k: int, n_extra: int, rows: int, H: int, w, valid, out,
                     stream=None) -> None:
    st = load().moe_reduce_pairs(_addr(slab, "slab", _F32), k, n_extra, rows, H,
                                 _addr(w, "w", _F32), _addr(valid, "valid", _MASK),
                                 _addr(out, "out", _BF16), _stream(stream))
    _check(st, "moe_reduce_pairs")


def moe_reduce_partials(slots, n_slots: int, rows: int, H: int, valid, out, stream=None) -> None:
    st = load().moe_reduce_partials(_addr(slots, "slots", _F32), n_slots, rows, H,
                                    _addr(valid, "valid", _MASK), _addr(out, "out", _BF16),
                                    _stream(stream))
    _check(st, "moe_reduce_partials")


def moe_route_from_logits(plan, logits, valid, T: int, k: int, topk_ids, topk_w, perm, offsets,
                          workspace, ws_bytes: int, stream=None) -> None:
    st = load().moe_route_from_logits(plan, _addr(logits, "logits", _F32),
                                      _addr(valid, "valid", _MASK), T, k,
                                      _addr(topk_ids, "topk_ids", _I32),
                                      _addr(topk_w, "topk_w", _F32), _addr(perm, "perm", _I32),
                                      _addr(offsets, "offsets", _I32),
                                      _addr(workspace, "workspace"), ws_bytes, _stream(stream))
    _check(st, "moe_route_from_logits")


def moe_route_from_logits_noalloc(plan, logits, valid, T: int, k: int, topk_ids, topk_w, perm,
                                  offsets, stream=None) -> None:
    """Routing from logits with the library's own static device scratch: for
    callers that cannot allocate device memory (no workspace argument)."""
    st = load().moe_route_from_logits_noalloc(plan, _addr(logits, "logits", _F32),
                                              _addr(valid, "valid", _MASK), T, k,
                                              _addr(topk_ids, "topk_ids", _I32),
                                              _addr(topk_w, "topk_w", _F32),
                                              _addr(perm, "perm", _I32),
                                              _addr(offsets, "offsets", _I32), _stream(stream))
    _check(st, "moe_route_from_logits_noalloc")


def moe_check_device_status(plan, workspace, stream=None) -> int:
    """Returns the device status bits (0 = none); synchronises the stream."""
    bits = ctypes.c_uint32()
    st = load().moe_check_device_status(plan, _addr(workspace, "workspace"), _stream(stream),
                                        ctypes.byref(bits))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoeError(st, "moe_check_device_status")
    return bits.value


def _host_addr(t, name: str, dtypes=None) -> int | None:
    """Address of a host (CPU) tensor argument: contiguous, of one of ``dtypes``."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if t.is_cuda:
        raise ValueError(f"{name}: a host tensor is required, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: a contiguous tensor is required")
    if dtypes is not None and str(t.dtype).rsplit(".", 1)[-1] not in dtypes:
        raise ValueError(f"{name}: element type {t.dtype} is not one of {', '.join(dtypes)}")
    return t.data_ptr()


def moe_pipeline_slot_bytes(plan, rows: int, depth: int) -> int:
    n = ctypes.c_size_t()
    _check(load().moe_pipeline_slot_bytes(plan, rows, depth, ctypes.byref(n)),
           "moe_pipeline_slot_bytes")
    return n.value


def moe_pipeline_create(plan, weights: moe_weights, k: int, rows: int, depth: int,
                        use_graph: bool, slots, slots_bytes: int, workspace, ws_bytes: int):
    h = _vp()
    _check(load().moe_pipeline_create(plan, ctypes.byref(weights), k, rows, depth,
                                      int(bool(use_graph)), _addr(slots, "slots"), slots_bytes,
                                      _addr(workspace, "workspace"), ws_bytes, ctypes.byref(h)),
           "moe_pipeline_create")
    return h.value


def moe_pipeline_submit(pipeline, hidden_host, valid_host, out_host) -> None:
    _check(load().moe_pipeline_submit(pipeline, _host_addr(hidden_host, "hidden_host", _BF16),
                                      _host_addr(valid_host, "valid_host", _MASK),
                                      _host_addr(out_host, "out_host", _BF16)),
           "moe_pipeline_submit")


def moe_pipeline_synchronize(pipeline) -> None:
    _check(load().moe_pipeline_synchronize(pipeline), "moe_pipeline_synchronize")


def moe_pipeline_streams(pipeline):
    """(upload, compute, download) cudaStream_t handles as ints."""
    u, c, d = _vp(), _vp(), _vp()
    _check(load().moe_pipeline_streams(pipeline, ctypes.byref(u), ctypes.byref(c),
                                       ctypes.byref(d)), "moe_pipeline_streams")
    return u.value or 0, c.value or 0, d.value or 0


def moe_pipeline_destroy(pipeline) -> None:
    load().moe_pipeline_destroy(pipeline)


def moe_get_workspace_views(plan, workspace) -> moe_workspace_views:
    v = moe_workspace_views()
    _check(load().moe_get_workspace_views(plan, _addr(workspace, "workspace"), ctypes.byref(v)),
           "moe_get_workspace_views")
    return v


class Plan:
    """A plan plus a torch-allocated workspace on the current device."""

    def __init__(self, *, max_tokens: int, hidden: int, num_experts: int, top_k_max: int,
                 inter: int, num_shared: int = 0, shared_inter: int = 0, renormalize: int = 1,
                 wtype: int = MOE_W_BF16, device=None):
        import torch
        self.cfg = moe_config(max_tokens, hidden, num_experts, top_k_max, inter, num_shared,
                              shared_inter, renormalize, wtype)
        self.handle, self.ws_bytes = moe_plan_create(self.cfg)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8,
                                     device=device if device is not None else "cuda")

    def weights(self, router_w, router_b=None, w_gate_up=None, w_down=None, s_gate_up=None,
                s_down=None, ws_gate_up=None, ws_down=None, ss_gate_up=None,
                ss_down=None, split_router=True, stream=None) -> moe_weights:
        """``make_weights`` with every tensor's shape checked against the plan: router
        [E, H] (+ bias [E]), gate/up [E, 2I, H], down [E, H, I], FP8 block scales
        [E, 2I/128, H/128] and [E, H/128, I/128], shared expert [2Is, H] / [H, Is] with
        scales [2Is/128, H/128] / [H/128, Is/128] (a mis-shaped tensor would be read
        past its end on the device).  Raw int addresses are taken as they are.
        With split_router, the router weights' bf16 split is made here once
        (moe_split_router_weights, on ``stream``) into a tensor the returned
        structure keeps alive, and forwards read it; make the weights again after
        changing router_w."""
        c = self.cfg
        E, H, I, Is = c.num_experts, c.hidden, c.inter, c.shared_inter
        fp8 = c.wtype == MOE_W_FP8_E4M3_B128
        want = {"router_w": (E, H), "w_gate_up": (E, 2 * I, H), "w_down": (E, H, I)}
        optional = {"router_b": (E,)}
        if fp8:
            want.update(s_gate_up=(E, 2 * I // 128, H // 128), s_down=(E, H // 128, I // 128))
        if c.num_shared:
            want.update(ws_gate_up=(2 * Is, H), ws_down=(H, Is))
            if fp8:
                want.update(ss_gate_up=(2 * Is // 128, H // 128), ss_down=(H // 128, Is // 128))
        given = dict(router_w=router_w, router_b=router_b, w_gate_up=w_gate_up, w_down=w_down,
                     s_gate_up=s_gate_up, s_down=s_down, ws_gate_up=ws_gate_up,
                     ws_down=ws_down, ss_gate_up=ss_gate_up, ss_down=ss_down)
        for name, shape in {**want, **optional}.items():
            t = given[name]
            if t is None:
                if name in want:
                    raise ValueError(f"{name} is required by this plan")
                continue
            if not isinstance(t, int) and tuple(t.shape) != shape:
                raise ValueError(f"{name}: shape {tuple(t.shape)}, the plan needs {shape}")
        if not split_router:
            return make_weights(**given)
        import torch
        nbytes = moe_router_split_bytes(self.handle)
        split = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=self.workspace.device)
        moe_split_router_weights(self.handle, router_w, split, nbytes, stream)
        w = make_weights(**given, router_split=split)
        w._router_split = split          # the structure holds only its address
        return w

    def _rows(self, hidden, valid, out=None) -> int:
        """T of a call, after checking hidden [T, H], valid [T] and out [T, H]."""
        H = self.cfg.hidden
        if hidden.dim() != 2 or hidden.shape[1] != H:
            raise ValueError(f"hidden: shape {tuple(hidden.shape)}, the plan needs [T, {H}]")
        T = hidden.shape[0]
        if valid is not None and tuple(valid.shape) != (T,):
            raise ValueError(f"valid: shape {tuple(valid.shape)}, needs ({T},)")
        if out is not None and tuple(out.shape) != (T, H):
            raise ValueError(f"out: shape {tuple(out.shape)}, needs ({T}, {H})")
        return T

    def _slabs(self, dst, rows: int):
        """Each receive slab tensor must hold len(dst) row blocks of ``rows`` rows."""
        need = len(dst) * rows * self.cfg.hidden
        for d in dst:
            if not isinstance(d, int) and d.numel() < need:
                raise ValueError(f"dst: a slab of {d.numel()} values, needs {need}")

    def forward(self, weights: moe_weights, hidden, valid, k: int, out, stream=None, dbg=None):
        moe_forward(self.handle, weights, hidden, valid, self._rows(hidden, valid, out), k, out,
                    self.workspace, self.ws_bytes, stream, dbg)

    def forward_scatter(self, weights: moe_weights, hidden, valid, k: int, dst,
                        rows_per_rank: int, slot: int, stream=None, dbg=None):
        T = self._rows(hidden, valid)
        self._slabs(dst, rows_per_rank)
        moe_forward_scatter(self.handle, weights, hidden, valid, T, k, dst,
                            rows_per_rank, slot, self.workspace, self.ws_bytes, stream, dbg)

    def forward_scatter_experts(self, weights: moe_weights, hidden, valid, k: int, dst,
                                rows_per_rank: int, slot: int, expert_begin: int,
                                expert_end: int, stream=None, dbg=None):
        T = self._rows(hidden, valid)
        self._slabs(dst, rows_per_rank)
        moe_forward_scatter_experts(self.handle, weights, hidden, valid, T, k, dst,
                                    rows_per_rank, slot, expert_begin, expert_end,
                                    self.workspace, self.ws_bytes, stream, dbg)

    def forward_scatter_pairs(self, weights: moe_weights, hidden, valid, k: int, dst,
                              rows_per_rank: int, shared_slot: int, expert_begin: int,
                              expert_end: int, send_ctas: int, stream=None, dbg=None):
        T = self._rows(hidden, valid)
        need = (k + 1) * rows_per_rank * self.cfg.hidden
        for d in dst:
            if not isinstance(d, int) and d.numel() < need:
                raise ValueError(f"dst: a slab of {d.numel()} values, needs at least {need}")
        moe_forward_scatter_pairs(self.handle, weights, hidden, valid, T, k, dst, rows_per_rank,
                                  shared_slot, expert_begin, expert_end, send_ctas,
                                  self.workspace, self.ws_bytes, stream, dbg)

    def route_from_logits(self, logits, valid, k: int, topk_ids, topk_w, perm, offsets,
                          stream=None):
        moe_route_from_logits(self.handle, logits, valid, logits.shape[0], k, topk_ids, topk_w,
                              perm, offsets, self.workspace, self.ws_bytes, stream)

    def device_status(self, stream=None) -> int:
        return moe_check_device_status(self.handle, self.workspace, stream)

    def views(self) -> moe_workspace_views:
        return moe_get_workspace_views(self.handle, self.workspace)

    def set_wait_limit(self, ns: int):
        moe_plan_set_wait_limit(self.handle, ns)

    def close(self):
        if self.handle:
            moe_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
