"""Thin Python binding of libmoonep (include/moonep.h): argument marshalling only.

Functions carry the C names.  Tensors are torch CUDA tensors; their data
pointers and the current CUDA stream are passed straight to the C ABI, and
every step of the hot path runs in the library's kernels.  There is no CPU
fallback: if the shared library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoonep.so")

OK, ERR_NULL, ERR_CONFIG, ERR_ALIGN, ERR_CUDA, ERR_SIZE, ERR_DEVICE = 0, -1, -2, -3, -4, -5, -6
STATUS_BAD_EXPERT, STATUS_DUP_EXPERT, STATUS_COUNT_MISMATCH, STATUS_BAD_PLAN, STATUS_TIMEOUT = 1, 2, 4, 8, 16
MAX_R, MAX_E, MAX_K, MAX_PROJ = 64, 4096, 32, 8
TRAINING, INFERENCE, INFERENCE_BY_COUNT, TRAINING_FEWEST_COPIES = 0, 1, 2, 3


class MoonepError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {error_string(code)} ({code})"
        if code == ERR_CUDA:
            msg += f" [{lib.moonep_last_error().decode()}]"
        super().__init__(msg)
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("S", "H", "K", "E", "R", "B", "token_padding", "num_sms", "mode")]


class PlanSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("dst", "cu_seqlens", "row_counts", "slot_expert", "counts", "assign", "maxvio", "status", "nvs")]


class IpcHandle(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_int64), ("bytes", ctypes.c_int64)]


class PlanStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dst", "cu_seqlens", "row_counts", "slot_expert", "counts", "assign", "maxvio", "status")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m load_balancing_planner_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "moonep_create": ([ctypes.POINTER(Config), ctypes.POINTER(P)], ctypes.c_int),
        "moonep_destroy": ([P], ctypes.c_int),
        "moonep_nvs": ([P], i64),
        "moonep_get_config": ([P, ctypes.POINTER(Config)], ctypes.c_int),
        "moonep_plan": ([P, P, P, ctypes.POINTER(PlanStruct), P], ctypes.c_int),
        "moonep_dispatch": ([P, ctypes.POINTER(PlanStruct), P, P, P, P, P], ctypes.c_int),
        "moonep_combine": ([P, ctypes.POINTER(PlanStruct), P, P, P, P, P], ctypes.c_int),
        "moonep_prefetch_weight": ([P, ctypes.POINTER(PlanStruct), i32, P, P, i64, P], ctypes.c_int),
        "moonep_reduce_grad": ([P, ctypes.POINTER(PlanStruct), i32, P, P, i64, P], ctypes.c_int),
        "moonep_read_status": ([ctypes.POINTER(PlanStruct), ctypes.POINTER(i32), P], ctypes.c_int),
        "moonep_plan_status": ([ctypes.POINTER(PlanStruct), ctypes.POINTER(i32)], ctypes.c_int),
        "moonep_plan_sizes": ([ctypes.POINTER(Config), i32, ctypes.POINTER(PlanSizes)], ctypes.c_int),
        "moonep_set_plan_barrier": ([P, ctypes.c_uint32, i32], ctypes.c_int),
        "moonep_ipc_export": ([P, ctypes.POINTER(IpcHandle)], ctypes.c_int),
        "moonep_ipc_import": ([ctypes.POINTER(IpcHandle), ctypes.POINTER(P)], ctypes.c_int),
        "moonep_ipc_close": ([P], ctypes.c_int),
        "moonep_error_string": ([ctypes.c_int], ctypes.c_char_p),
        "moonep_last_error": ([], ctypes.c_char_p),
        "moonep_plan_noalloc": ([ctypes.POINTER(Config), P, P, ctypes.POINTER(PlanStruct), P], ctypes.c_int),
        "moonep_group_gemm": ([P, ctypes.POINTER(PlanStruct), P, P, P, P, i64, P], ctypes.c_int),
        "moonep_plan_rank": ([P, i32, P, P, ctypes.POINTER(PlanStruct), P], ctypes.c_int),
        "moonep_dispatch_rank": ([P, ctypes.POINTER(PlanStruct), P, P, P, P, P], ctypes.c_int),
        "moonep_combine_rank": ([P, ctypes.POINTER(PlanStruct), P, P, P, P, P], ctypes.c_int),
        "moonep_prefetch_weight_rank": ([P, ctypes.POINTER(PlanStruct), i32, i32, P, P, i64, P], ctypes.c_int),
        "moonep_reduce_grad_rank": ([P, ctypes.POINTER(PlanStruct), i32, i32, P, P, i64, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()
EXPORTS = ("moonep_create", "moonep_destroy", "moonep_nvs", "moonep_get_config", "moonep_plan",
           "moonep_dispatch", "moonep_combine", "moonep_prefetch_weight", "moonep_reduce_grad",
           "moonep_read_status", "moonep_error_string", "moonep_last_error", "moonep_plan_noalloc",
           "moonep_group_gemm", "moonep_plan_rank", "moonep_dispatch_rank", "moonep_combine_rank",
           "moonep_prefetch_weight_rank", "moonep_reduce_grad_rank", "moonep_plan_sizes", "moonep_plan_status",
           "moonep_set_plan_barrier", "moonep_ipc_export", "moonep_ipc_import", "moonep_ipc_close")
NOALLOC_SCRATCH_BYTES = 1 << 20


def error_string(code: int) -> str:
    return lib.moonep_error_string(code).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise MoonepError(rc, what)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("moonep takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("moonep takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t, shape, dtype, name):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name}: expected {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")


class Handle:
    """Owns a moonep_handle_t (and its planning workspace)."""

    def __init__(self, ptr: int, cfg: Config):
        self.ptr = ctypes.c_void_p(ptr)
        self.cfg = cfg
        self.nvs = int(lib.moonep_nvs(self.ptr))

    def __getattr__(self, k):
        if k in ("S", "H", "K", "E", "R", "B", "token_padding", "num_sms", "mode"):
            return getattr(self.cfg, k)
        raise AttributeError(k)

    def close(self):
        if self.ptr:
            _check(lib.moonep_destroy(self.ptr), "moonep_destroy")
            self.ptr = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Plan:
    """Device arrays of one plan (caller-owned, see moonep_plan_t).  `h` is a
    Handle, or a Config for moonep_plan_noalloc.  `rank` marks one rank's
    plan (moonep_plan_rank): dst is then [S,K]."""

    def __init__(self, h, device=None, rank: int | None = None):
        dev = device or torch.device("cuda", torch.cuda.current_device())
        R, S, K, E, B = h.R, h.S, h.K, h.E, h.B
        # element counts from the C ABI (moonep_plan_sizes), viewed in the
        # arrays' documented shapes
        sz = moonep_plan_sizes(h.cfg if isinstance(h, Handle) else h, rank is not None)
        i32 = dict(dtype=torch.int32, device=dev)
        self.rank = rank
        self.dst = torch.empty(sz.dst, **i32).view((S, K) if rank is not None else (R, S, K))
        self.cu_seqlens = torch.empty(sz.cu_seqlens, **i32).view(R, E + B)
        self.row_counts = torch.empty(sz.row_counts, **i32).view(R, E + B)
        self.slot_expert = torch.empty(max(sz.slot_expert, R), **i32).view(R, max(B, 1))
        self.counts = torch.empty(sz.counts, **i32).view(R, E)
        self.assign = torch.empty(sz.assign, **i32).view(R, 4)
        self.maxvio = torch.empty(sz.maxvio, dtype=torch.float32, device=dev)
        self.status = torch.zeros(sz.status, **i32)
        self.struct = PlanStruct(*(t.data_ptr() for t in (
            self.dst, self.cu_seqlens, self.row_counts, self.slot_expert, self.counts,
            self.assign, self.maxvio, self.status)))
        self.nvs = h.nvs if isinstance(h, Handle) else None
        self.B = B

    def slots(self):
        return self.slot_expert[:, : self.B]


def moonep_plan_sizes(cfg: Config, one_rank: bool = False) -> PlanSizes:
    """Element counts of the plan arrays for cfg (and NvS), from the C ABI."""
    out = PlanSizes()
    _check(lib.moonep_plan_sizes(ctypes.byref(cfg), 1 if one_rank else 0, ctypes.byref(out)), "moonep_plan_sizes")
    return out


def moonep_set_plan_barrier(h: "Handle", max_polls: int = 0, missing: int = 0):
    """Test hook: the planner's grid barrier of h gives up after max_polls
    polls and waits for `missing` arrivals that never come ((0, 0) = normal)."""
    _check(lib.moonep_set_plan_barrier(h.ptr, max_polls, missing), "moonep_set_plan_barrier")


def moonep_ipc_export(t) -> bytes:
    """The CUDA IPC export of the allocation holding CUDA tensor t (plain
    bytes, to send to another process)."""
    h = IpcHandle()
    _check(lib.moonep_ipc_export(_ptr(t), ctypes.byref(h)), "moonep_ipc_export")
    return ctypes.string_at(ctypes.addressof(h), ctypes.sizeof(h))


def moonep_ipc_import(blob: bytes) -> int:
    """Device pointer, in this process, of another process's export."""
    if len(blob) != ctypes.sizeof(IpcHandle):
        raise ValueError("not a moonep IPC handle")
    h = IpcHandle.from_buffer_copy(blob)
    out = ctypes.c_void_p()
    _check(lib.moonep_ipc_import(ctypes.byref(h), ctypes.byref(out)), "moonep_ipc_import")
    return int(out.value)


def moonep_ipc_close(ptr: int):
    _check(lib.moonep_ipc_close(ctypes.c_void_p(ptr)), "moonep_ipc_close")


def moonep_create(S, H, K, E, R, B=None, token_padding=128, num_sms=0, mode=TRAINING) -> Handle:
    B = E // R if B is None else B
    cfg = Config(S, H, K, E, R, B, token_padding, num_sms, mode)
    out = ctypes.c_void_p()
    _check(lib.moonep_create(ctypes.byref(cfg), ctypes.byref(out)), "moonep_create")
    return Handle(out.value, cfg)


def moonep_destroy(h: Handle):
    h.close()


def moonep_nvs(h: Handle) -> int:
    return int(lib.moonep_nvs(h.ptr))


def moonep_plan(h: Handle, topk, tokens_per_expert=None, plan: Plan | None = None, stream=None) -> Plan:
    _expect(topk, (h.R, h.S, h.K), torch.int32, "topk")
    _expect(tokens_per_expert, (h.R, h.E), torch.int32, "tokens_per_expert")
    plan = plan or Plan(h, topk.device)
    _check(lib.moonep_plan(h.ptr, _ptr(topk), _ptr(tokens_per_expert), ctypes.byref(plan.struct),
                           _stream(stream)), "moonep_plan")
    return plan


def moonep_plan_noalloc(cfg: Config, topk, tokens_per_expert=None, plan: Plan | None = None,
                        stream=None) -> Plan:
    """The planner without a handle or any device allocation (see moonep.h)."""
    _expect(topk, (cfg.R, cfg.S, cfg.K), torch.int32, "topk")
    _expect(tokens_per_expert, (cfg.R, cfg.E), torch.int32, "tokens_per_expert")
    plan = plan or Plan(cfg, topk.device)
    _check(lib.moonep_plan_noalloc(ctypes.byref(cfg), _ptr(topk), _ptr(tokens_per_expert),
                                   ctypes.byref(plan.struct), _stream(stream)), "moonep_plan_noalloc")
    return plan


def _group_plan(plan: Plan, what: str):
    if plan.rank is not None:
        raise ValueError(f"{what} takes a group plan; use the _rank call with a rank's plan")


def _rank_plan(plan: Plan, what: str):
    if plan.rank is None:
        raise ValueError(f"{what} takes a plan from moonep_plan_rank")


def moonep_plan_rank(h: Handle, rank: int, topk, counts_all, plan: Plan | None = None, stream=None) -> Plan:
    """One rank's plan from its own picks topk [S,K] and every rank's router
    counts counts_all [R,E] (row q = rank q's tokens_per_expert)."""
    _expect(topk, (h.S, h.K), torch.int32, "topk")
    _expect(counts_all, (h.R, h.E), torch.int32, "counts_all")
    plan = plan or Plan(h, topk.device, rank=rank)
    _rank_plan(plan, "moonep_plan_rank")
    plan.rank = rank
    _check(lib.moonep_plan_rank(h.ptr, rank, _ptr(topk), _ptr(counts_all), ctypes.byref(plan.struct),
                                _stream(stream)), "moonep_plan_rank")
    return plan


def moonep_dispatch_rank(h: Handle, plan: Plan, hidden, route_weights, hidden_nvs, route_weights_nvs=None,
                         stream=None):
    """Scatter one rank's rows hidden [S,H] (and route_weights [S,K]) into the
    R ranks' buffers: hidden_nvs is a list (or PeerTable) of R [NvS,H] bf16
    tensors, route_weights_nvs None or a list (or PeerTable) of R [NvS] fp32
    tensors."""
    _rank_plan(plan, "moonep_dispatch_rank")
    _expect(hidden, (h.S, h.H), torch.bfloat16, "hidden")
    _expect(route_weights, (h.S, h.K), torch.float32, "route_weights")
    bufs, wbufs = _rank_tables(h, hidden_nvs, route_weights_nvs)
    _check(lib.moonep_dispatch_rank(h.ptr, ctypes.byref(plan.struct), _ptr(hidden), _ptr(route_weights),
                                    bufs, wbufs, _stream(stream)), "moonep_dispatch_rank")


def moonep_combine_rank(h: Handle, plan: Plan, hidden_nvs, route_weights_nvs=None, out=None,
                        gathered_weights=None, gather=True, stream=None):
    """out [S,H] = the weighted sum of each own token's K slots, read from the
    R ranks' buffers (lists as in moonep_dispatch_rank)."""
    _rank_plan(plan, "moonep_combine_rank")
    bufs, wbufs = _rank_tables(h, hidden_nvs, route_weights_nvs)
    dev = torch.device("cuda", torch.cuda.current_device())
    if out is None:
        out = torch.empty((h.S, h.H), dtype=torch.bfloat16, device=dev)
    if gather and route_weights_nvs is not None and gathered_weights is None:
        gathered_weights = torch.empty((h.S, h.K), dtype=torch.float32, device=dev)
    _expect(out, (h.S, h.H), torch.bfloat16, "out")
    _expect(gathered_weights, (h.S, h.K), torch.float32, "gathered_weights")
    _check(lib.moonep_combine_rank(h.ptr, ctypes.byref(plan.struct), bufs, wbufs, _ptr(out),
                                   _ptr(gathered_weights), _stream(stream)), "moonep_combine_rank")
    return out, gathered_weights


class PeerTable:
    """The R ranks' same-shaped tensors as one table of device pointers,
    checked once.  Pass it wherever a per-rank call takes a list of R
    tensors: the call then skips the per-tensor checks and the marshalling.
    The table keeps the tensors alive; their storage must not move.  An entry
    may also be a plain device pointer (int), e.g. a peer process's buffer
    mapped with moonep_ipc_import, assumed to hold `shape` of `dtype`."""

    def __init__(self, tensors, shape, dtype, name="table"):
        self.tensors = list(tensors)
        for t in self.tensors:
            _expect_entry(t, shape, dtype, name)
        self.arr = _ptr_array(self.tensors)
        self.shape, self.dtype, self.name = tuple(shape), dtype, name

    def __len__(self):
        return len(self.tensors)

    def __getitem__(self, i):
        return self.tensors[i]


def _expect_entry(t, shape, dtype, name):
    """A table entry: a tensor of `shape` and `dtype`, or a device pointer (int)."""
    if isinstance(t, int):
        if t == 0 or t % 16:
            raise ValueError(f"{name}: a device pointer must be non-zero and 16-byte aligned")
        return
    _expect(t, shape, dtype, name)


def _table(h: Handle, x, shape, dtype, name):
    if x is None:
        return None
    if isinstance(x, PeerTable):
        if len(x) != h.R or x.shape != tuple(shape) or x.dtype != dtype:
            raise ValueError(f"{name}: a table of {h.R} {tuple(shape)} {dtype} tensors expected")
        return x.arr
    if len(x) != h.R:
        raise ValueError("one buffer per rank")
    for b in x:
        _expect_entry(b, shape, dtype, name)
    return _ptr_array(x)


def _rank_tables(h: Handle, hidden_nvs, route_weights_nvs):
    return (_table(h, hidden_nvs, (h.nvs, h.H), torch.bfloat16, "hidden_nvs[q]"),
            _table(h, route_weights_nvs, (h.nvs,), torch.float32, "route_weights_nvs[q]"))


def moonep_dispatch(h: Handle, plan: Plan, hidden, route_weights=None, hidden_nvs=None,
                    route_weights_nvs=None, stream=None):
    _group_plan(plan, "moonep_dispatch")
    _expect(hidden, (h.R, h.S, h.H), torch.bfloat16, "hidden")
    _expect(route_weights, (h.R, h.S, h.K), torch.float32, "route_weights")
    if hidden_nvs is None:
        hidden_nvs = torch.empty((h.R, h.nvs, h.H), dtype=torch.bfloat16, device=hidden.device)
    if route_weights is not None and route_weights_nvs is None:
        route_weights_nvs = torch.empty((h.R, h.nvs), dtype=torch.float32, device=hidden.device)
    _expect(hidden_nvs, (h.R, h.nvs, h.H), torch.bfloat16, "hidden_nvs")
    _expect(route_weights_nvs, (h.R, h.nvs), torch.float32, "route_weights_nvs")
    _check(lib.moonep_dispatch(h.ptr, ctypes.byref(plan.struct), _ptr(hidden), _ptr(route_weights),
                               _ptr(hidden_nvs), _ptr(route_weights_nvs), _stream(stream)), "moonep_dispatch")
    return hidden_nvs, route_weights_nvs


def moonep_combine(h: Handle, plan: Plan, hidden_nvs, route_weights_nvs=None, out=None,
                   gathered_weights=None, gather=True, stream=None):
    _group_plan(plan, "moonep_combine")
    _expect(hidden_nvs, (h.R, h.nvs, h.H), torch.bfloat16, "hidden_nvs")
    _expect(route_weights_nvs, (h.R, h.nvs), torch.float32, "route_weights_nvs")
    if out is None:
        out = torch.empty((h.R, h.S, h.H), dtype=torch.bfloat16, device=hidden_nvs.device)
    if gather and route_weights_nvs is not None and gathered_weights is None:
        gathered_weights = torch.empty((h.R, h.S, h.K), dtype=torch.float32, device=hidden_nvs.device)
    _expect(out, (h.R, h.S, h.H), torch.bfloat16, "out")
    _expect(gathered_weights, (h.R, h.S, h.K), torch.float32, "gathered_weights")
    _check(lib.moonep_combine(h.ptr, ctypes.byref(plan.struct), _ptr(hidden_nvs), _ptr(route_weights_nvs),
                              _ptr(out), _ptr(gathered_weights), _stream(stream)), "moonep_combine")
    return out, gathered_weights


def _ptr_array(ts):
    """A C array of device pointers: tensors' data pointers, or ints as given."""
    for t in ts:
        if not isinstance(t, int) and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("moonep takes contiguous CUDA tensors")
    return (ctypes.c_void_p * len(ts))(*[t if isinstance(t, int) else t.data_ptr() for t in ts])


def moonep_prefetch_weight(h: Handle, plan: Plan, weights, pool, stream=None):
    """weights: list of [E, H, Hp] bf16; pool: list of [R, B, H, Hp] bf16."""
    if len(weights) != len(pool) or not weights:
        raise ValueError("one pool per weight tensor")
    Hp = weights[0].shape[-1]
    for W, P in zip(weights, pool):
        _expect(W, (h.E, h.H, Hp), torch.bfloat16, "weights")
        _expect(P, (h.R, h.B, h.H, Hp), torch.bfloat16, "pool")
    _check(lib.moonep_prefetch_weight(h.ptr, ctypes.byref(plan.struct), len(weights), _ptr_array(weights),
                                      _ptr_array(pool), Hp, _stream(stream)), "moonep_prefetch_weight")


def moonep_reduce_grad(h: Handle, plan: Plan, grads, reduce_buffers, stream=None):
    """grads: list of [E, H, Hp] fp32; reduce_buffers: list of [R, B, H, Hp] fp32."""
    if len(grads) != len(reduce_buffers) or not grads:
        raise ValueError("one reduce buffer per grad tensor")
    Hp = grads[0].shape[-1]
    for G, RB in zip(grads, reduce_buffers):
        _expect(G, (h.E, h.H, Hp), torch.float32, "grads")
        _expect(RB, (h.R, h.B, h.H, Hp), torch.float32, "reduce_buffers")
    _check(lib.moonep_reduce_grad(h.ptr, ctypes.byref(plan.struct), len(grads), _ptr_array(grads),
                                  _ptr_array(reduce_buffers), Hp, _stream(stream)), "moonep_reduce_grad")


def _rank_weight_tables(h: Handle, own, peers, own_shape, peer_shape, dtype, names):
    if not own or len(own) != len(peers) or any(len(row) != h.R for row in peers):
        raise ValueError(f"one {names[0]} per projection and one {names[1]} per rank and projection")
    Hp = own[0].shape[-1]
    for t in own:
        _expect(t, (*own_shape, h.H, Hp), dtype, names[0])
    for row in peers:
        for t in row:
            _expect_entry(t, (*peer_shape, h.H, Hp), dtype, names[1])
    return _ptr_array(own), _ptr_array([t for row in peers for t in row]), Hp


def moonep_prefetch_weight_rank(h: Handle, plan: Plan, rank: int, weights, pool, stream=None):
    """One rank's prefetch: weights[p][q] is rank q's home experts [G,H,Hp]
    bf16 of projection p, pool[p] this rank's slots [B,H,Hp] bf16."""
    G = h.E // h.R
    own, peers, Hp = _rank_weight_tables(h, list(pool), [list(r) for r in weights], (h.B,), (G,),
                                         torch.bfloat16, ("pool", "weights"))
    _check(lib.moonep_prefetch_weight_rank(h.ptr, ctypes.byref(plan.struct), rank, len(pool), peers, own, Hp,
                                           _stream(stream)), "moonep_prefetch_weight_rank")


def moonep_reduce_grad_rank(h: Handle, plan: Plan, rank: int, grads, reduce_buffers, stream=None):
    """One home rank's reduction: grads[p] is its home experts' [G,H,Hp] fp32
    gradients, reduce_buffers[p][q] rank q's slots [B,H,Hp] fp32."""
    G = h.E // h.R
    own, peers, Hp = _rank_weight_tables(h, list(grads), [list(r) for r in reduce_buffers], (G,), (h.B,),
                                         torch.float32, ("grads", "reduce_buffers"))
    _check(lib.moonep_reduce_grad_rank(h.ptr, ctypes.byref(plan.struct), rank, len(grads), own, peers, Hp,
                                       _stream(stream)), "moonep_reduce_grad_rank")


def moonep_group_gemm(h: Handle, plan: Plan, x_nvs, weights, pool=None, y_nvs=None, stream=None):
    """y_nvs [R,NvS,Hp] = x_nvs rows of each plan row @ that row's expert
    weight (weights [E,H,Hp] bf16 for rows < E, pool [R,B,H,Hp] bf16 for
    slot rows)."""
    Hp = weights.shape[-1]
    _expect(x_nvs, (h.R, h.nvs, h.H), torch.bfloat16, "x_nvs")
    _expect(weights, (h.E, h.H, Hp), torch.bfloat16, "weights")
    _expect(pool, (h.R, h.B, h.H, Hp), torch.bfloat16, "pool")
    if y_nvs is None:
        y_nvs = torch.empty((h.R, h.nvs, Hp), dtype=torch.bfloat16, device=x_nvs.device)
    _expect(y_nvs, (h.R, h.nvs, Hp), torch.bfloat16, "y_nvs")
    _check(lib.moonep_group_gemm(h.ptr, ctypes.byref(plan.struct), _ptr(x_nvs), _ptr(weights), _ptr(pool),
                                 _ptr(y_nvs), Hp, _stream(stream)), "moonep_group_gemm")
    return y_nvs


def moonep_plan_status(plan: Plan) -> int:
    """plan.status after waiting for all work on the current device."""
    st = ctypes.c_int32(0)
    _check(lib.moonep_plan_status(ctypes.byref(plan.struct), ctypes.byref(st)), "moonep_plan_status")
    return int(st.value)


def moonep_read_status(plan: Plan, stream=None) -> int:
    st = ctypes.c_int32(0)
    _check(lib.moonep_read_status(ctypes.byref(plan.struct), ctypes.byref(st), _stream(stream)),
           "moonep_read_status")
    return int(st.value)
