"""Query-aware sparse attention over a long KV cache on B200 (sm_100a).

Thin Python binding of ``libspa.so`` (the C ABI in ``include/spa.h``).  Every function
here only marshals torch tensors into pointers, sizes and the current CUDA stream and
calls the library; every step of the computation runs in the library's CUDA kernels.
There is no fallback: if ``libspa.so`` is missing or a call fails, an exception is raised.

Output tensors and workspaces are allocated here through torch (the caller's allocator);
the library itself never allocates device memory.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from ._abi import (SPA_COLLAPSE_GROUP_MEAN, SPA_COLLAPSE_NONE, SPA_DECODE_AUTO, SPA_DECODE_FUSED, SPA_DECODE_SEPARATE,
                   SPA_SCORE_LOWRANK, SPA_SCORE_MEAN_BLOCK,
                   SPA_SCORE_MINMAX_BLOCK, SPA_SCORE_TAYLOR_BLOCK, SPA_SELECT_TOPK, SPA_STATS_BF16, SPA_SELECT_TOPP, SpaDecodeArgs, SpaError, SpaPbsArgs, SpaPrefillArgs, check, lib, lib_path)

__all__ = [
    "SpaError", "lib", "lib_path", "block_stats", "index_scores", "select_topk", "select_topp", "sparse_attend",
    "decode", "DecodePlan", "workspace", "read_device_status", "select_topp_static", "prefill", "PrefillPlan", "SPA_COLLAPSE_NONE", "SPA_COLLAPSE_GROUP_MEAN",
    "SPA_SCORE_LOWRANK", "SPA_SCORE_TAYLOR_BLOCK", "SPA_SCORE_MINMAX_BLOCK", "SPA_SCORE_MEAN_BLOCK",
    "SPA_SELECT_TOPK", "SPA_SELECT_TOPP", "SPA_STATS_BF16", "block_minmax", "rla_state",
    "SPA_DECODE_AUTO", "SPA_DECODE_SEPARATE", "SPA_DECODE_FUSED", "pbs_prefill", "PbsPlan",
]


def _stream(stream: Optional[torch.cuda.Stream] = None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled device workspace of nbytes (uint8)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def read_device_status(ws: torch.Tensor, reset: bool = True) -> int:
    """Device status bits of a workspace (1 << SPA_ERR_* for each condition raised)."""
    bits = ctypes.c_uint32(0)
    check(lib().spa_read_device_status(ctypes.c_void_p(ws.data_ptr()), _stream(), ctypes.byref(bits), int(reset)))
    return bits.value


# ----------------------------------------------------------------------------- a1
def block_stats(K: torch.Tensor, block: int = 64, bf16: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """K [B, Hkv, N, d] bf16 -> (mean, var) [B, Hkv, N // block, d], fp32 (or bf16 storage)."""
    _need(K, torch.bfloat16, "K")
    B, Hkv, N, d = K.shape
    nb = N // block
    mean = torch.empty((B, Hkv, nb, d), dtype=torch.bfloat16 if bf16 else torch.float32, device=K.device)
    var = torch.empty_like(mean)
    fn = lib().spa_block_stats_bf16 if bf16 else lib().spa_block_stats
    check(fn(_ptr(K), B, Hkv, N, d, block, _ptr(mean), _ptr(var), _stream()))
    return mean, var


def block_minmax(K: torch.Tensor, block: int = 64, bf16: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """K [B, Hkv, N, d] bf16 -> per-block channel (min, max) [B, Hkv, N // block, d], fp32 (or bf16)."""
    _need(K, torch.bfloat16, "K")
    B, Hkv, N, d = K.shape
    nb = N // block
    mn = torch.empty((B, Hkv, nb, d), dtype=torch.bfloat16 if bf16 else torch.float32, device=K.device)
    mx = torch.empty_like(mn)
    fn = lib().spa_block_minmax_bf16 if bf16 else lib().spa_block_minmax
    check(fn(_ptr(K), B, Hkv, N, d, block, _ptr(mn), _ptr(mx), _stream()))
    return mn, mx


# ----------------------------------------------------------------------------- a2/a3
def index_scores(kind: int, q: torch.Tensor, keys: torch.Tensor, var: Optional[torch.Tensor], Hkv: int,
                 collapse: int, scale: float, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Scores [U, M] fp32.  LOWRANK: q = q_idx [B, Hq, 16] bf16, keys = Kidx [B, Hkv, M, 16] bf16.
    TAYLOR: q [B, Hq, d] bf16, keys = block means [B, Hkv, M, d] fp32, var likewise.
    MINMAX: keys = block minima, var = block maxima.  MEAN: keys = block means, var None."""
    _need(q, torch.bfloat16, "q")
    B, Hq, dim = q.shape
    M = keys.shape[2]
    if kind == SPA_SCORE_LOWRANK:
        _need(keys, torch.bfloat16, "keys")
    else:
        sdt = torch.bfloat16 if kind & SPA_STATS_BF16 else torch.float32
        _need(keys, sdt, "keys")
        if kind & ~SPA_STATS_BF16 != SPA_SCORE_MEAN_BLOCK:
            _need(var, sdt, "var")
    U = B * (Hkv if collapse == SPA_COLLAPSE_GROUP_MEAN else Hq)
    if out is None:
        out = torch.empty((U, M), dtype=torch.float32, device=q.device)
    check(lib().spa_index_scores(kind, _ptr(q), _ptr(keys), _ptr(var), B, Hq, Hkv, M, dim, collapse,
                                 ctypes.c_float(scale), _ptr(out), _stream()))
    return out


# ----------------------------------------------------------------------------- a4-a6
def _select_out(U: int, cap: int, device) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    idx = torch.full((U, max(cap, 1)), -1, dtype=torch.int32, device=device)
    count = torch.zeros(U, dtype=torch.int32, device=device)
    ws = workspace(lib().spa_select_workspace_bytes(U, 0), device)
    return idx, count, ws


def select_topk(scores: torch.Tensor, k: int, sink: int, window: int, cap: Optional[int] = None,
                unit_len: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """scores [U, M] fp32 -> (idx [U, cap] int32 ascending, count [U] int32)."""
    _need(scores, torch.float32, "scores")
    if unit_len is not None:
        _need(unit_len, torch.int32, "unit_len")
    U, M = scores.shape
    cap = min(M, k + sink + window) if cap is None else cap
    idx, count, ws = _select_out(U, cap, scores.device)
    check(lib().spa_select_topk(_ptr(scores), _ptr(unit_len), U, M, k, sink, window, _ptr(idx), _ptr(count), cap,
                                _ptr(ws), ws.numel(), _stream()))
    return idx, count


def select_topp(scores: torch.Tensor, p: float, sink: int, window: int, cap: Optional[int] = None,
                unit_len: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """scores [U, M] fp32 -> (idx [U, cap] int32 ascending, count [U] int32, index_mass [U] fp32)."""
    _need(scores, torch.float32, "scores")
    if unit_len is not None:
        _need(unit_len, torch.int32, "unit_len")
    U, M = scores.shape
    cap = M if cap is None else cap
    idx, count, ws = _select_out(U, cap, scores.device)
    mass = torch.zeros(U, dtype=torch.float32, device=scores.device)
    check(lib().spa_select_topp(_ptr(scores), _ptr(unit_len), U, M, ctypes.c_float(p), sink, window, _ptr(idx),
                                _ptr(count), cap, _ptr(mass), _ptr(ws), ws.numel(), _stream()))
    return idx, count, mass


def select_topp_static(scores: torch.Tensor, p: float, sink: int, window: int, cap: Optional[int] = None,
                       unit_len: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """select_topp without a workspace: for callers that may not allocate device memory when
    they call (outputs must then be preallocated by them; here they are allocated for
    convenience).  The library keeps the scratch in a fixed device array shared by all calls,
    so calls must not overlap on the GPU; at most SPA_SELECT_STATIC_MAX_UNITS units."""
    _need(scores, torch.float32, "scores")
    if unit_len is not None:
        _need(unit_len, torch.int32, "unit_len")
    U, M = scores.shape
    cap = M if cap is None else cap
    idx = torch.full((U, max(cap, 1)), -1, dtype=torch.int32, device=scores.device)
    count = torch.zeros(U, dtype=torch.int32, device=scores.device)
    mass = torch.zeros(U, dtype=torch.float32, device=scores.device)
    check(lib().spa_select_topp_static(_ptr(scores), _ptr(unit_len), U, M, ctypes.c_float(p), sink, window,
                                       _ptr(idx), _ptr(count), cap, _ptr(mass), _stream()))
    return idx, count, mass


# ----------------------------------------------------------------------------- a7/a8
def sparse_attend(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, idx: torch.Tensor, count: torch.Tensor,
                  collapse: int, sm_scale: float, unit_tokens: int = 1, ws: Optional[torch.Tensor] = None,
                  want_f32: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor], torch.Tensor]:
    """q [B, Hq, d], K/V [B, Hkv, N, d] bf16; idx [U, cap], count [U] int32 ->
    (out [B, Hq, d] bf16, out_f32 [B, Hq, d] or None, lse [B, Hq] fp32)."""
    for t, n in ((q, "q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n)
    _need(idx, torch.int32, "idx")
    _need(count, torch.int32, "count")
    B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    out32 = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device) if want_f32 else None
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(lib().spa_attend_workspace_bytes(B, Hq, Hkv, d, collapse), q.device)
    check(lib().spa_sparse_attend(_ptr(q), _ptr(K), _ptr(V), B, Hq, Hkv, N, d, _ptr(idx), _ptr(count),
                                  idx.shape[1], collapse, unit_tokens, ctypes.c_float(sm_scale), _ptr(out),
                                  _ptr(out32), _ptr(lse), _ptr(ws), ws.numel(), _stream()))
    return out, out32, lse


# ----------------------------------------------------------------------------- fused decode
@dataclass
class DecodePlan:
    """Arguments, outputs and workspace of one fused decode step, built once and reused."""

    args: SpaDecodeArgs
    ws: torch.Tensor
    idx: torch.Tensor
    count: torch.Tensor
    index_mass: Optional[torch.Tensor]
    out: torch.Tensor
    out_f32: Optional[torch.Tensor]
    lse: Optional[torch.Tensor]
    keep: tuple   # tensors the pointers refer to

    def run(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        check(lib().spa_decode(ctypes.byref(self.args), ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(),
                               _stream(stream)))

    @property
    def fused(self) -> bool:
        """Whether spa_decode runs these arguments as the fused persistent kernel."""
        return lib().spa_decode_path_taken(ctypes.byref(self.args)) == SPA_DECODE_FUSED

    def run_timed(self, events, stream: Optional[torch.cuda.Stream] = None) -> None:
        """run() recording four torch.cuda.Event (enable_timing=True, already recorded once so that
        they exist) before scoring, after scoring, after selection and after attention."""
        handles = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
        check(lib().spa_decode_timed(ctypes.byref(self.args), ctypes.c_void_p(self.ws.data_ptr()),
                                     self.ws.numel(), _stream(stream), handles))


def decode(*, score_kind: int, select_kind: int, collapse: int, q: torch.Tensor, K: torch.Tensor,
           V: torch.Tensor, q_idx: Optional[torch.Tensor] = None, Kidx: Optional[torch.Tensor] = None,
           bmean: Optional[torch.Tensor] = None, bvar: Optional[torch.Tensor] = None, block: int = 1,
           score_scale: float, sm_scale: float, topk: int = 0, topp: float = 0.0, sink: int = 0,
           window: int = 0, cap: Optional[int] = None, want_f32: bool = True, want_lse: bool = True,
           local_units: Optional[torch.Tensor] = None, rla_state: Optional[torch.Tensor] = None,
           rla_z: Optional[torch.Tensor] = None, rla_gamma: Optional[torch.Tensor] = None,
           rla_eps: float = 1e-6, kernel_path: int = SPA_DECODE_AUTO, run: bool = True) -> DecodePlan:
    """Build (and by default run) a fused decode step; see spa_decode in include/spa.h.
    local_units: optional uint8 [U] on the device, nonzero for the units that head-wise routing
    makes local (support = sink + window, not scored).
    rla_state / rla_z / rla_gamma: optional fp32 [B, Hkv, d, d] / [B, Hkv, d] / [Hq, d] that
    add the residual linear attention over the rows outside each support (state from
    rla_state()).
    kernel_path: SPA_DECODE_AUTO / SPA_DECODE_SEPARATE (scoring, selection and attention as
    separate kernels) or SPA_DECODE_FUSED (the persistent dataflow kernel where it applies)."""
    for t, n in ((q, "q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n)
    B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    U = B * (Hkv if collapse == SPA_COLLAPSE_GROUP_MEAN else Hq)
    M = N // block
    if cap is None:
        cap = min(M, topk + sink + window) if select_kind == SPA_SELECT_TOPK else M
    dev = q.device
    idx = torch.full((U, max(cap, 1)), -1, dtype=torch.int32, device=dev)
    count = torch.zeros(U, dtype=torch.int32, device=dev)
    mass = torch.zeros(U, dtype=torch.float32, device=dev) if select_kind == SPA_SELECT_TOPP else None
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    out32 = torch.empty((B, Hq, d), dtype=torch.float32, device=dev) if want_f32 else None
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev) if want_lse else None
    a = SpaDecodeArgs()
    a.score_kind, a.select_kind, a.collapse = score_kind, select_kind, collapse
    a.B, a.Hq, a.Hkv, a.N, a.d = B, Hq, Hkv, N, d
    a.r = q_idx.shape[-1] if q_idx is not None else 16
    a.block = block
    a.q, a.K, a.V = _ptr(q), _ptr(K), _ptr(V)
    a.q_idx, a.Kidx = _ptr(q_idx), _ptr(Kidx)
    a.bmean, a.bvar = _ptr(bmean), _ptr(bvar)
    a.stats_bf16 = int(bmean is not None and bmean.dtype == torch.bfloat16)
    a.score_scale, a.sm_scale = score_scale, sm_scale
    a.topk, a.topp, a.sink, a.window = topk, topp, sink, window
    a.kernel_path = kernel_path
    a.idx, a.count, a.cap = _ptr(idx), _ptr(count), cap
    a.index_mass = _ptr(mass)
    a.out, a.out_f32, a.lse = _ptr(out), _ptr(out32), _ptr(lse)
    if local_units is not None:
        _need(local_units, torch.uint8, "local_units")
        if local_units.numel() != U:
            raise ValueError(f"local_units must hold one flag per unit ({U})")
    a.local_units = _ptr(local_units)
    if rla_state is not None:
        for t, n, shape in ((rla_state, "rla_state", (B, Hkv, d, d)), (rla_z, "rla_z", (B, Hkv, d)),
                            (rla_gamma, "rla_gamma", (Hq, d))):
            if t is None:
                raise ValueError(f"{n} is required with rla_state")
            _need(t, torch.float32, n)
            if tuple(t.shape) != shape:
                raise ValueError(f"{n} must have shape {shape}, got {tuple(t.shape)}")
        a.rla_state, a.rla_z, a.rla_gamma, a.rla_eps = _ptr(rla_state), _ptr(rla_z), _ptr(rla_gamma), rla_eps
    ws = workspace(lib().spa_decode_workspace_bytes(ctypes.byref(a)), dev)
    plan = DecodePlan(a, ws, idx, count, mass, out, out32, lse,
                      (q, K, V, q_idx, Kidx, bmean, bvar, local_units, rla_state, rla_z, rla_gamma))
    if run:
        plan.run()
    return plan


# ----------------------------------------------------------------------------- RLA state
def rla_state(K: torch.Tensor, V: torch.Tensor, S: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
              n0: int = 0, n1: Optional[int] = None, stream: Optional[torch.cuda.Stream] = None):
    """Add rows [n0, n1) of K, V [B, Hkv, N, d] bf16 into the residual-linear-attention state
    S [B, Hkv, d, d], z [B, Hkv, d] (fp32, zero-filled when not given); see spa_rla_state
    in include/spa.h.  Returns (S, z)."""
    _need(K, torch.bfloat16, "K")
    _need(V, torch.bfloat16, "V")
    B, Hkv, N, d = K.shape
    if tuple(V.shape) != (B, Hkv, N, d):
        raise ValueError("K and V must have the same shape")
    S = torch.zeros((B, Hkv, d, d), dtype=torch.float32, device=K.device) if S is None else S
    z = torch.zeros((B, Hkv, d), dtype=torch.float32, device=K.device) if z is None else z
    _need(S, torch.float32, "S")
    _need(z, torch.float32, "z")
    if tuple(S.shape) != (B, Hkv, d, d) or tuple(z.shape) != (B, Hkv, d):
        raise ValueError("S must be [B, Hkv, d, d] and z [B, Hkv, d]")
    n1 = N if n1 is None else n1
    check(lib().spa_rla_state(_ptr(K), _ptr(V), B, Hkv, N, d, n0, n1, _ptr(S), _ptr(z), _stream(stream)),
          "spa_rla_state")
    return S, z


# ----------------------------------------------------------------------------- a9 shared-support prefill
@dataclass
class PrefillPlan:
    """Arguments, outputs and workspace of one shared-support prefill call, reusable."""

    args: SpaPrefillArgs
    ws: torch.Tensor
    idx: torch.Tensor
    count: torch.Tensor
    out: torch.Tensor
    out_f32: Optional[torch.Tensor]
    keep: tuple

    per_query: bool = False

    def run(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        fn = lib().spa_prefill_per_query if self.per_query else lib().spa_prefill_shared
        check(fn(ctypes.byref(self.args), ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(), _stream(stream)))

    def run_timed(self, events, stream: Optional[torch.cuda.Stream] = None) -> None:
        """run() of the shared-support prefill recording two torch.cuda.Event (enable_timing=True,
        already recorded once) right before and right after its attention kernel."""
        if self.per_query:
            raise ValueError("run_timed times the shared-support prefill's attention kernel")
        handles = (ctypes.c_void_p * 2)(*[ctypes.c_void_p(e.cuda_event) for e in events])
        check(lib().spa_prefill_shared_timed(ctypes.byref(self.args), ctypes.c_void_p(self.ws.data_ptr()),
                                             self.ws.numel(), _stream(stream), handles))


def prefill(*, Q: torch.Tensor, q_idx: torch.Tensor, K: torch.Tensor, V: torch.Tensor, Kidx: torch.Tensor,
            q_start: int, score_scale: float, sm_scale: float, topk: int, sink: int, bq: int = 64,
            want_f32: bool = True, run: bool = True) -> PrefillPlan:
    """Sparse prefill of one query chunk.  bq = 64: one support per 64 queries
    (spa_prefill_shared in include/spa.h); bq = 1: one support per query
    (spa_prefill_per_query; idx[u][count[u]] then holds the query's own position).
    Q [T, Hq, d], q_idx [T, Hq, r], K/V [Hkv, N, d], Kidx [Hkv, N, r], all bf16."""
    for t, n in ((Q, "Q"), (q_idx, "q_idx"), (K, "K"), (V, "V"), (Kidx, "Kidx")):
        _need(t, torch.bfloat16, n)
    T, Hq, d = Q.shape
    Hkv, N, _ = K.shape
    U = (T // bq) * Hkv
    per_query = bq == 1
    cap = min(N, topk + sink) + (1 if per_query else 0)
    dev = Q.device
    idx = torch.full((U, max(cap, 1)), -1, dtype=torch.int32, device=dev)
    count = torch.zeros(U, dtype=torch.int32, device=dev)
    out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=dev)
    out32 = torch.empty((T, Hq, d), dtype=torch.float32, device=dev) if want_f32 else None
    a = SpaPrefillArgs()
    a.T, a.Hq, a.Hkv, a.N, a.d, a.r = T, Hq, Hkv, N, d, q_idx.shape[-1]
    a.q_start, a.bq = q_start, bq
    a.Q, a.q_idx, a.K, a.V, a.Kidx = _ptr(Q), _ptr(q_idx), _ptr(K), _ptr(V), _ptr(Kidx)
    a.score_scale, a.sm_scale = score_scale, sm_scale
    a.topk, a.sink = topk, sink
    a.idx, a.count, a.cap = _ptr(idx), _ptr(count), cap
    a.out, a.out_f32 = _ptr(out), _ptr(out32)
    nbytes = (lib().spa_prefill_per_query_workspace_bytes if per_query else lib().spa_prefill_workspace_bytes)(
        ctypes.byref(a))
    ws = workspace(nbytes, dev)
    plan = PrefillPlan(a, ws, idx, count, out, out32, (Q, q_idx, K, V, Kidx), per_query)
    if run:
        plan.run()
    return plan


# ----------------------------------------------------------------------------- PBS-Attn prefill
@dataclass
class PbsPlan:
    """Arguments, outputs and workspace of one permuted block-sparse prefill, reusable."""

    args: SpaPbsArgs
    ws: torch.Tensor
    importance: torch.Tensor
    perm: torch.Tensor
    idx: torch.Tensor
    count: torch.Tensor
    out: torch.Tensor
    out_f32: Optional[torch.Tensor]
    keep: tuple

    def run(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        check(lib().spa_pbs_prefill(ctypes.byref(self.args), ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(),
                                    _stream(stream)))

    def run_timed(self, events, stream: Optional[torch.cuda.Stream] = None) -> None:
        """run() recording two torch.cuda.Event (enable_timing=True, already recorded once) right
        before and right after the attention kernel."""
        handles = (ctypes.c_void_p * 2)(*[ctypes.c_void_p(e.cuda_event) for e in events])
        check(lib().spa_pbs_prefill_timed(ctypes.byref(self.args), ctypes.c_void_p(self.ws.data_ptr()),
                                          self.ws.numel(), _stream(stream), handles))


def pbs_prefill(*, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, sm_scale: float, S: int, topk: int,
                b: int = 64, want_f32: bool = True, run: bool = True) -> PbsPlan:
    """Permuted block-sparse prefill of a causal sequence; see spa_pbs_prefill in include/spa.h.
    Q [T, Hq, d], K/V [Hkv, T, d] bf16."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n)
    T, Hq, d = Q.shape
    Hkv = K.shape[0]
    U = (T // b) * Hkv
    cap = max(topk * b, 1)
    dev = Q.device
    imp = torch.empty((Hkv, T), dtype=torch.float32, device=dev)
    perm = torch.empty((Hkv, T), dtype=torch.int32, device=dev)
    idx = torch.full((U, cap), -1, dtype=torch.int32, device=dev)
    count = torch.zeros(U, dtype=torch.int32, device=dev)
    out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=dev)
    out32 = torch.empty((T, Hq, d), dtype=torch.float32, device=dev) if want_f32 else None
    a = SpaPbsArgs()
    a.T, a.Hq, a.Hkv, a.d, a.b, a.S, a.topk, a.sm_scale = T, Hq, Hkv, d, b, S, topk, sm_scale
    a.Q, a.K, a.V = _ptr(Q), _ptr(K), _ptr(V)
    a.importance, a.perm, a.idx, a.count, a.cap = _ptr(imp), _ptr(perm), _ptr(idx), _ptr(count), cap
    a.out, a.out_f32 = _ptr(out), _ptr(out32)
    ws = workspace(lib().spa_pbs_workspace_bytes(ctypes.byref(a)), dev)
    plan = PbsPlan(a, ws, imp, perm, idx, count, out, out32, (Q, K, V))
    if run:
        plan.run()
    return plan
