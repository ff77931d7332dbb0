"""Spava / APB-V approximate-attention prefill on B200 (sm_100a), all hosts virtual.

A thin Python binding over the C ABI of ``libspava.so`` (include/spava.h): it checks
tensor dtypes, shapes, devices and contiguity and passes raw device pointers and
the current CUDA stream.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and every entry point raises if the
library is missing or the call fails.

Layouts: q [N+T, hq, d], k/v [N+T, hkv, d] bf16; o like q; lse [hq, N+T] fp32;
scores [hkv, N] fp32; idx [H-1, hkv, P] int32; passing K/V [hkv, H-1, P, d] bf16.
"""

import ctypes
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import SpavaError, load  # noqa: F401

__all__ = ["Plan", "score_select", "gather_passing", "attn_prefill", "attn_prefill_two_stage", "dense_causal",
           "check_device_error", "SpavaError", "load", "last_launch_count", "shard_owners", "shard_stage",
           "layer_workspace", "qkv_projection", "out_projection", "check_layer_error"]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t: torch.Tensor, name: str, dtype, shape, device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


class Plan:
    """Sizes of one prefill layer plus its device-side work lists (spava_plan)."""

    def __init__(self, n_visual: int, n_text: int, n_hosts: int,
                 host_sizes: Optional[Sequence[int]], anchor: int, passing: int, probe_r: int,
                 hq: int, hkv: int, head_dim: int, softmax_scale: float = 0.0,
                 device: Optional[torch.device] = None):
        self.lib = _lib.load()
        self.n_visual, self.n_text, self.n_hosts = int(n_visual), int(n_text), int(n_hosts)
        self.anchor, self.passing, self.probe_r = int(anchor), int(passing), int(probe_r)
        self.hq, self.hkv, self.head_dim = int(hq), int(hkv), int(head_dim)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        sizes = None
        if host_sizes is not None:
            arr = (ctypes.c_int32 * len(host_sizes))(*[int(x) for x in host_sizes])
            sizes = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
        handle = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            st = self.lib.spava_plan_create(ctypes.byref(handle), self.n_visual, self.n_text,
                                            self.n_hosts, sizes, self.anchor, self.passing,
                                            self.probe_r, self.hq, self.hkv, self.head_dim,
                                            ctypes.c_float(softmax_scale))
        _lib.check(st, "spava_plan_create")
        self._h = handle
        self.workspace_bytes = int(self.lib.spava_workspace_bytes(self._h))
        self.two_stage_workspace_bytes = int(self.lib.spava_two_stage_workspace_bytes(self._h))
        off = (ctypes.c_int32 * (self.n_hosts + 1))()
        self.lib.spava_plan_offsets(self._h, off)
        self.offsets = [int(x) for x in off]

    @property
    def handle(self):
        return self._h

    @property
    def n_total(self) -> int:
        return self.n_visual + self.n_text

    def new_workspace(self, two_stage: bool = False) -> torch.Tensor:
        n = self.two_stage_workspace_bytes if two_stage else self.workspace_bytes
        return torch.zeros(max(n, 256), dtype=torch.uint8, device=self.device)

    SCORE_REDUCE = {"max": 0, "sum": 1, "mean": 2, "per_query_head": 3}

    def set_score_reduce(self, mode: str) -> None:
        """spava_plan_set_score_reduce: how the query heads of a KV group combine the
        probe scores ("max" default, "sum", "mean" of the per-head maxima), or
        "per_query_head": every query head selects its own passing keys.  Call before
        new_workspace: the selection rows set the workspace size."""
        if mode not in self.SCORE_REDUCE:
            raise ValueError(f"score reduction must be one of {sorted(self.SCORE_REDUCE)}")
        _lib.check(self.lib.spava_plan_set_score_reduce(self._h, self.SCORE_REDUCE[mode]), "spava_plan_set_score_reduce")
        self.score_reduce = mode
        self._refresh_sizes()

    SCORE_KIND = {"logit": 0, "prob": 1}

    def set_score_kind(self, kind: str) -> None:
        """spava_plan_set_score_kind: "logit" (default) or "prob" (each probe row's
        attention probability over its own block).  Call before new_workspace."""
        if kind not in self.SCORE_KIND:
            raise ValueError(f"score kind must be one of {sorted(self.SCORE_KIND)}")
        _lib.check(self.lib.spava_plan_set_score_kind(self._h, self.SCORE_KIND[kind]), "spava_plan_set_score_kind")
        self.score_kind = kind
        self._refresh_sizes()

    def set_fused_select(self, enable: bool) -> None:
        """spava_plan_set_fused_select: True scores, selects and gathers in one persistent
        launch where the plan allows it; False (default) runs the score kernel, then
        select+gather."""
        _lib.check(self.lib.spava_plan_set_fused_select(self._h, int(bool(enable))), "spava_plan_set_fused_select")

    def _refresh_sizes(self) -> None:
        self.workspace_bytes = int(self.lib.spava_workspace_bytes(self._h))
        self.two_stage_workspace_bytes = int(self.lib.spava_two_stage_workspace_bytes(self._h))
        if getattr(self, "shard_world", 0):
            self.shard_workspace_bytes = int(self.shard_layout().workspace_bytes)

    def set_shard(self, rank: int, world: int, owner: Sequence[int]) -> None:
        """spava_plan_set_shard: this plan runs rank ``rank`` of ``world``, host h on rank
        owner[h] (the same list on every rank).  Query shard_layout() afterwards."""
        if len(owner) != self.n_hosts:
            raise ValueError(f"owner needs one rank per host ({self.n_hosts})")
        arr = (ctypes.c_int32 * self.n_hosts)(*[int(x) for x in owner])
        with torch.cuda.device(self.device):
            _lib.check(self.lib.spava_plan_set_shard(self._h, int(rank), int(world), arr), "spava_plan_set_shard")
        self.shard_rank, self.shard_world, self.owner = int(rank), int(world), [int(x) for x in owner]
        self._refresh_sizes()

    def shard_owners(self, world: int, policy: str = "zigzag"):
        """spava_plan_shard_owners: the rank of every host; "longest_first" balances this
        plan's per-host costs (uneven blocks), the others as shard_owners()."""
        if policy not in SHARD_POLICY:
            raise ValueError(f"policy must be one of {sorted(SHARD_POLICY)}")
        arr = (ctypes.c_int32 * self.n_hosts)()
        _lib.check(self.lib.spava_plan_shard_owners(self._h, int(world), SHARD_POLICY[policy], arr),
                   "spava_plan_shard_owners")
        return [int(x) for x in arr]

    def shard_layout(self) -> "_lib.ShardLayout":
        """spava_shard_query: byte offsets of the exchange buffers in the sharded workspace."""
        out = _lib.ShardLayout()
        _lib.check(self.lib.spava_shard_query(self._h, ctypes.byref(out)), "spava_shard_query")
        return out

    def shard_stage(self, stage: int, q, k, v, o, lse, workspace: torch.Tensor, stream=None) -> None:
        """spava_shard_stage (module function shard_stage) on this plan."""
        shard_stage(self, stage, q, k, v, o, lse, workspace, stream)

    def set_debug(self, wait_limit_ns: int = 0, stall_producer: bool = False) -> None:
        _lib.check(self.lib.spava_plan_set_debug(self._h, int(wait_limit_ns), int(bool(stall_producer))),
                   "spava_plan_set_debug")

    # kernel timing hook (spava_profile_*)
    def profile_begin(self, max_marks: int = 4096) -> None:
        _lib.check(self.lib.spava_profile_begin(self._h, int(max_marks)), "spava_profile_begin")

    def profile_read(self, max_entries: int = 4096):
        """[(kernel name, ms), ...] of the kernels recorded since the last read."""
        labels = (ctypes.c_int32 * max_entries)()
        ms = (ctypes.c_float * max_entries)()
        n = self.lib.spava_profile_read(self._h, labels, ms, max_entries)
        if n < 0:
            raise SpavaError(3, "spava_profile_read", "event query failed")
        return [(self.lib.spava_kernel_name(labels[i]).decode(), float(ms[i])) for i in range(n)]

    def profile_end(self) -> None:
        _lib.check(self.lib.spava_profile_end(self._h), "spava_profile_end")

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.check(self.lib.spava_plan_destroy(self._h), "spava_plan_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # shape helpers
    def qkv_shapes(self):
        NT = self.n_total
        return (NT, self.hq, self.head_dim), (NT, self.hkv, self.head_dim)

    @property
    def score_rows(self) -> int:
        """Selection rows: KV heads, or query heads with per-query-head selection."""
        return self.hq if getattr(self, "score_reduce", "max") == "per_query_head" else self.hkv

    def scores_shape(self):
        return (self.score_rows, self.n_visual)

    def idx_shape(self):
        return (max(self.n_hosts - 1, 0), self.score_rows, self.passing)

    def pass_shape(self):
        return (self.score_rows, max(self.n_hosts - 1, 0), self.passing, self.head_dim)

    def _check_qkv(self, q, k, v=None):
        qs, ks = self.qkv_shapes()
        _expect(q, "q", torch.bfloat16, qs, self.device)
        _expect(k, "k", torch.bfloat16, ks, self.device)
        if v is not None:
            _expect(v, "v", torch.bfloat16, ks, self.device)


def _ws(plan: Plan, workspace: Optional[torch.Tensor], two_stage: bool = False) -> torch.Tensor:
    if workspace is None:
        workspace = plan.new_workspace(two_stage)
    need = plan.two_stage_workspace_bytes if two_stage else plan.workspace_bytes
    if workspace.dtype != torch.uint8 or workspace.numel() < need or \
            workspace.device != plan.device or workspace.data_ptr() % 256:
        raise ValueError(f"workspace: uint8, 256-byte aligned, >= {need} bytes on the plan's device")
    return workspace


def score_select(plan: Plan, q: Optional[torch.Tensor], k: Optional[torch.Tensor],
                 scores: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                 scores_given: bool = False, workspace: Optional[torch.Tensor] = None, stream=None):
    """spava_score_select: probe scores [hkv, N] fp32 and passing indices [H-1, hkv, P]."""
    dev = plan.device
    if scores_given:
        _expect(scores, "scores", torch.float32, plan.scores_shape(), dev)
    else:
        plan._check_qkv(q, k)
        if scores is None:
            scores = torch.empty(plan.scores_shape(), dtype=torch.float32, device=dev)
        _expect(scores, "scores", torch.float32, plan.scores_shape(), dev)
    if idx is None:
        idx = torch.empty(plan.idx_shape(), dtype=torch.int32, device=dev)
    _expect(idx, "idx", torch.int32, plan.idx_shape(), dev)
    ws = _ws(plan, workspace)
    st = plan.lib.spava_score_select(plan.handle, _ptr(q), _ptr(k), _ptr(scores), _ptr(idx),
                                     _lib.SPAVA_SCORES_GIVEN if scores_given else 0, _ptr(ws),
                                     _stream(stream))
    _lib.check(st, "spava_score_select")
    return scores, idx


def gather_passing(plan: Plan, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                   k_pass: Optional[torch.Tensor] = None, v_pass: Optional[torch.Tensor] = None,
                   stream=None):
    """spava_gather_passing: passing K/V [hkv, H-1, P, d] gathered from k/v by idx."""
    _, ks = plan.qkv_shapes()
    _expect(k, "k", torch.bfloat16, ks, plan.device)
    _expect(v, "v", torch.bfloat16, ks, plan.device)
    _expect(idx, "idx", torch.int32, plan.idx_shape(), plan.device)
    if k_pass is None:
        k_pass = torch.empty(plan.pass_shape(), dtype=torch.bfloat16, device=plan.device)
    if v_pass is None:
        v_pass = torch.empty(plan.pass_shape(), dtype=torch.bfloat16, device=plan.device)
    _expect(k_pass, "k_pass", torch.bfloat16, plan.pass_shape(), plan.device)
    _expect(v_pass, "v_pass", torch.bfloat16, plan.pass_shape(), plan.device)
    st = plan.lib.spava_gather_passing(plan.handle, _ptr(k), _ptr(v), _ptr(idx), _ptr(k_pass),
                                       _ptr(v_pass), _stream(stream))
    _lib.check(st, "spava_gather_passing")
    return k_pass, v_pass


def attn_prefill(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 scores_out: Optional[torch.Tensor] = None, idx_out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """spava_attn_prefill: the whole approximate-attention prefill of one layer.

    Returns (o [N+T, hq, d] bf16, lse [hq, N+T] fp32)."""
    plan._check_qkv(q, k, v)
    dev = plan.device
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((plan.hq, plan.n_total), dtype=torch.float32, device=dev)
    _expect(o, "o", torch.bfloat16, tuple(q.shape), dev)
    _expect(lse, "lse", torch.float32, (plan.hq, plan.n_total), dev)
    if scores_out is not None:
        _expect(scores_out, "scores_out", torch.float32, plan.scores_shape(), dev)
    if idx_out is not None:
        _expect(idx_out, "idx_out", torch.int32, plan.idx_shape(), dev)
    ws = _ws(plan, workspace)
    st = plan.lib.spava_attn_prefill(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     _ptr(scores_out), _ptr(idx_out), _ptr(ws), _stream(stream))
    _lib.check(st, "spava_attn_prefill")
    return o, lse


def attn_prefill_two_stage(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                           scores_out: Optional[torch.Tensor] = None, idx_out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None, stream=None):
    """spava_attn_prefill_two_stage: the prefill as local pass (with fused probe scores)
    -> select/gather -> remote pass merged through the lse.  Needs the larger
    plan.two_stage_workspace_bytes workspace."""
    plan._check_qkv(q, k, v)
    dev = plan.device
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((plan.hq, plan.n_total), dtype=torch.float32, device=dev)
    _expect(o, "o", torch.bfloat16, tuple(q.shape), dev)
    _expect(lse, "lse", torch.float32, (plan.hq, plan.n_total), dev)
    if scores_out is not None:
        _expect(scores_out, "scores_out", torch.float32, plan.scores_shape(), dev)
    if idx_out is not None:
        _expect(idx_out, "idx_out", torch.int32, plan.idx_shape(), dev)
    ws = _ws(plan, workspace, two_stage=True)
    st = plan.lib.spava_attn_prefill_two_stage(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                               _ptr(scores_out), _ptr(idx_out), _ptr(ws), _stream(stream))
    _lib.check(st, "spava_attn_prefill_two_stage")
    return o, lse


def dense_causal(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """spava_dense_causal: dense causal attention over all N+T tokens."""
    plan._check_qkv(q, k, v)
    dev = plan.device
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((plan.hq, plan.n_total), dtype=torch.float32, device=dev)
    _expect(o, "o", torch.bfloat16, tuple(q.shape), dev)
    _expect(lse, "lse", torch.float32, (plan.hq, plan.n_total), dev)
    ws = _ws(plan, workspace)
    st = plan.lib.spava_dense_causal(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     _ptr(ws), _stream(stream))
    _lib.check(st, "spava_dense_causal")
    return o, lse


SHARD_POLICY = {"contiguous": _lib.SPAVA_SHARD_CONTIGUOUS, "zigzag": _lib.SPAVA_SHARD_ZIGZAG,
                "longest_first": _lib.SPAVA_SHARD_LONGEST_FIRST}


def shard_owners(n_hosts: int, world: int, policy: str = "zigzag"):
    """spava_shard_owners (host-side, no device): the rank of every host under the
    "contiguous" or "zigzag" policy ("longest_first" needs the plan: Plan.shard_owners)."""
    if policy not in SHARD_POLICY:
        raise ValueError(f"policy must be one of {sorted(SHARD_POLICY)}")
    lib = _lib.load()
    arr = (ctypes.c_int32 * max(int(n_hosts), 1))()
    _lib.check(lib.spava_shard_owners(int(n_hosts), int(world), SHARD_POLICY[policy], arr), "spava_shard_owners")
    return [int(arr[h]) for h in range(int(n_hosts))]


def shard_stage(plan: Plan, stage: int, q: Optional[torch.Tensor], k: Optional[torch.Tensor],
                v: Optional[torch.Tensor], o: Optional[torch.Tensor], lse: Optional[torch.Tensor],
                workspace: torch.Tensor, stream=None) -> None:
    """spava_shard_stage: one stage (SPAVA_SHARD_SELECT / LOCAL / REMOTE / MERGE, or
    ATTEND in place of LOCAL + REMOTE) of the sharded prefill on full-size q/k/v/o/lse
    buffers; see include/spava.h for which rows each stage reads and writes."""
    dev = plan.device
    if stage != _lib.SPAVA_SHARD_MERGE:
        plan._check_qkv(q, k, v)
    if stage != _lib.SPAVA_SHARD_SELECT:
        _expect(o, "o", torch.bfloat16, (plan.n_total, plan.hq, plan.head_dim), dev)
        _expect(lse, "lse", torch.float32, (plan.hq, plan.n_total), dev)
    need = getattr(plan, "shard_workspace_bytes", None)
    if need is None:
        raise ValueError("plan is not sharded (Plan.set_shard)")
    if workspace.dtype != torch.uint8 or workspace.numel() < need or workspace.device != dev or \
            workspace.data_ptr() % 256:
        raise ValueError(f"workspace: uint8, 256-byte aligned, >= {need} bytes on the plan's device")
    st = plan.lib.spava_shard_stage(plan.handle, int(stage), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                    _ptr(workspace), _stream(stream))
    _lib.check(st, "spava_shard_stage")


def check_device_error(plan: Plan, workspace: torch.Tensor, stream=None) -> None:
    """Synchronise and raise SpavaError(SPAVA_ERR_TIMEOUT) if a bounded device wait ran out."""
    _lib.check(plan.lib.spava_check_device_error(plan.handle, _ptr(workspace), _stream(stream)),
               "spava_check_device_error")


def last_launch_count() -> int:
    return int(_lib.load().spava_last_launch_count())


# ---------------------------------------------------------------- layer projections
def layer_workspace(n_tokens: int, device=None) -> torch.Tensor:
    """Workspace of spava_qkv_projection / spava_out_projection for n_tokens rows."""
    n = int(_lib.load().spava_layer_workspace_bytes(int(n_tokens)))
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=dev)


def _check_layer_ws(ws: torch.Tensor, n_tokens: int, device) -> None:
    need = int(_lib.load().spava_layer_workspace_bytes(int(n_tokens)))
    if ws.dtype != torch.uint8 or ws.numel() < need or ws.device != device or ws.data_ptr() % 256:
        raise ValueError(f"layer workspace: uint8, 256-byte aligned, >= {need} bytes on {device}")


def qkv_projection(x: torch.Tensor, w_qkv: torch.Tensor, hq: int, hkv: int, head_dim: int,
                   q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, workspace: torch.Tensor,
                   rms_eps: float = 1e-6, stream=None) -> None:
    """q, k, v = split((x / rms(x)) w_qkv^T) on the tensor cores (spava_qkv_projection).
    x [T, hidden], w_qkv [(hq + 2 hkv) head_dim, hidden], q [T, hq, head_dim],
    k/v [T, hkv, head_dim]: bf16, contiguous, on one device."""
    if x.dim() != 2:
        raise ValueError("x must be [tokens, hidden]")
    T, hidden = x.shape
    dev = x.device
    _expect(x, "x", torch.bfloat16, (T, hidden), dev)
    _expect(w_qkv, "w_qkv", torch.bfloat16, ((hq + 2 * hkv) * head_dim, hidden), dev)
    _expect(q, "q", torch.bfloat16, (T, hq, head_dim), dev)
    _expect(k, "k", torch.bfloat16, (T, hkv, head_dim), dev)
    _expect(v, "v", torch.bfloat16, (T, hkv, head_dim), dev)
    _check_layer_ws(workspace, T, dev)
    st = _lib.load().spava_qkv_projection(_ptr(x), T, hidden, _ptr(w_qkv), hq, hkv, head_dim, float(rms_eps),
                                          _ptr(q), _ptr(k), _ptr(v), _ptr(workspace), _stream(stream))
    _lib.check(st, "spava_qkv_projection")


def out_projection(o: torch.Tensor, w_o: torch.Tensor, x: torch.Tensor, workspace: torch.Tensor,
                   stream=None) -> None:
    """x += o w_o^T in place on the tensor cores (spava_out_projection).  o [T, ...]
    read as [T, in_features], w_o [hidden, in_features], x [T, hidden]: bf16."""
    T, hidden = x.shape
    dev = x.device
    in_features = o.numel() // max(T, 1)
    _expect(o.view(T, in_features), "o", torch.bfloat16, (T, in_features), dev)
    _expect(w_o, "w_o", torch.bfloat16, (hidden, in_features), dev)
    _expect(x, "x", torch.bfloat16, (T, hidden), dev)
    _check_layer_ws(workspace, T, dev)
    st = _lib.load().spava_out_projection(_ptr(o), T, in_features, _ptr(w_o), hidden, _ptr(x), _ptr(workspace),
                                          _stream(stream))
    _lib.check(st, "spava_out_projection")


def check_layer_error(workspace: torch.Tensor, stream=None) -> None:
    """Synchronise and raise SpavaError(SPAVA_ERR_TIMEOUT) if a projection's bounded wait ran out."""
    _lib.check(_lib.load().spava_layer_check_error(_ptr(workspace), _stream(stream)), "spava_layer_check_error")
