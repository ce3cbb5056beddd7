"""Python binding of libsas_b200.so -- SAS gated block-sparse attention on B200 (sm_100a).

Argument marshalling only: every step runs in the library's CUDA kernels; PyTorch
provides device memory and the current stream. The entry points carry the C names
(see include/sas.h for the operator, layouts and error behaviour). There is no CPU
path: without the compiled library, importing this package fails.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsas_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python gated_block_sparse_sas_b200/build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

SAS_OK, SAS_ERR_INVALID_ARG, SAS_ERR_UNSUPPORTED, SAS_ERR_CUDA, SAS_ERR_WORKSPACE = 0, -1, -2, -3, -4
SAS_BF16, SAS_FP32 = 0, 1
_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t


class SasProblem(ctypes.Structure):
    _fields_ = [("batch", _i32), ("total_tokens", _i32), ("max_seqlen", _i32),
                ("num_q_heads", _i32), ("num_kv_heads", _i32), ("head_dim", _i32),
                ("block", _i32), ("topk", _i32), ("gate_hidden", _i32), ("rms_eps", _f32),
                ("dtype", ctypes.c_int), ("cu_seqlens", _vp), ("gate_rope_cos", _vp),
                ("gate_rope_sin", _vp), ("gate_heads", _i32)]


class SasDecodeProblem(ctypes.Structure):
    _fields_ = [("batch", _i32), ("capacity", _i32), ("num_q_heads", _i32),
                ("num_kv_heads", _i32), ("head_dim", _i32), ("block", _i32), ("topk", _i32),
                ("gate_hidden", _i32), ("rms_eps", _f32), ("dtype", ctypes.c_int),
                ("seqlens", _vp), ("gate_rope_cos", _vp), ("gate_rope_sin", _vp),
                ("ungated", _i32), ("gate_heads", _i32)]


_P = ctypes.POINTER(SasProblem)
_DP = ctypes.POINTER(SasDecodeProblem)
_SIGS = {
    "sas_last_error": ([], ctypes.c_char_p),
    "sas_kernel_launches": ([], ctypes.c_uint64),
    "sas_rope_tables": ([_i32, _i32, ctypes.c_double, _vp, _vp], ctypes.c_int),
    "sas_pool_keys": ([_P, _vp, _vp, _vp], ctypes.c_int),
    "sas_gate_keys": ([_P, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "sas_gate_scores_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
    "sas_gate_scores": ([_P] + [_vp] * 9 + [_vp, _sz, _vp], ctypes.c_int),
    "sas_topk": ([_P, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "sas_gate_select_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
    "sas_gate_select": ([_P] + [_vp] * 10 + [_vp, _sz, _vp], ctypes.c_int),
    "sas_gate_bwd_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
    "sas_gate_bwd": ([_P] + [_vp] * 13 + [_vp, _sz, _vp], ctypes.c_int),
    "sas_attn_fwd_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
    "sas_attn_fwd": ([_P] + [_vp] * 8 + [_sz, _vp], ctypes.c_int),
    "sas_attn_bwd_workspace_size": ([_P, ctypes.POINTER(_sz)], ctypes.c_int),
    "sas_attn_bwd": ([_P] + [_vp] * 13 + [_sz, _vp], ctypes.c_int),
    "sas_decode_workspace_size": ([_DP, ctypes.POINTER(_sz)], ctypes.c_int),
    "sas_decode": ([_DP] + [_vp] * 14 + [_sz, _vp], ctypes.c_int),
    "sas_decode_paged": ([_DP, _vp, _i32] + [_vp] * 14 + [_sz, _vp], ctypes.c_int),
    "sas_decode_noalloc": ([_DP] + [_vp] * 13 + [_vp], ctypes.c_int),
    "sas_decode_noalloc_error_word": ([ctypes.POINTER(_vp)], ctypes.c_int),
    "sas_decode_set_fused": ([_i32], ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class SasError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {_lib.sas_last_error().decode()}")


def _check(status: int, where: str):
    if status != SAS_OK:
        raise SasError(status, where)


# Device-side error codes written to word 0 of a workspace (include/sas.h, "Device-side errors").
ERROR_CODES = {
    41: "decode attention: a bounded wait gave up",
    51: "attn_fwd: a bounded wait gave up", 52: "attn_fwd: a bounded wait gave up",
    53: "attn_fwd: a bounded wait gave up", 54: "attn_fwd: a bounded wait gave up",
    55: "attn_fwd: a bounded wait gave up", 56: "attn_fwd: a bounded wait gave up",
    57: "attn_fwd: a bounded wait gave up",
    60: "attn_fwd: a row's largest logit exceeds its own key's by more than ~97 nats",
    61: "decode: a row's largest logit exceeds its own key's by more than ~97 nats",
    62: "paged decode: a page id out of range",
    71: "attn_bwd: a bounded wait gave up", 72: "attn_bwd: a bounded wait gave up",
    73: "attn_bwd: a bounded wait gave up", 74: "attn_bwd: a bounded wait gave up",
    75: "attn_bwd: a bounded wait gave up", 76: "attn_bwd: a bounded wait gave up",
    77: "attn_bwd: a bounded wait gave up", 78: "attn_bwd: a bounded wait gave up",
    79: "attn_bwd: a bounded wait gave up",
    81: "decode attention: a bounded wait gave up", 82: "decode attention: a bounded wait gave up",
    83: "decode attention: a bounded wait gave up",
    84: "fused decode: a selection waited too long for its gate projections",
    85: "fused decode: an attention split waited too long for its selection",
    86: "fused decode: a bounded wait for cached gate keys gave up",
    91: "gate projections: a bounded wait gave up", 92: "gate projections: a bounded wait gave up",
    93: "gate projections: a bounded wait gave up",
    94: "router weight gradients: a bounded wait gave up",
    95: "router weight gradients: a bounded wait gave up",
    96: "router weight gradients: a bounded wait gave up",
    97: "tensor-core gate scores: a bounded wait gave up",
    98: "tensor-core gate scores: a bounded wait gave up",
    99: "tensor-core gate scores: a bounded wait gave up",
}


class SasDeviceError(RuntimeError):
    """A kernel reported a device-side failure through a workspace's error word."""

    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: device error code {code}: "
                         f"{ERROR_CODES.get(code, 'unknown code')}")


def error_code(workspace) -> int:
    """Word 0 of a workspace after its call: 0, or the device-side error code. Reading it
    waits for the work queued so far on the workspace's device."""
    return int(workspace[:4].view(torch.int32).item())


def check_workspace(workspace, where: str = "sas"):
    """Raise SasDeviceError if the call that used `workspace` reported a device-side error."""
    code = error_code(workspace)
    if code != 0:
        raise SasDeviceError(code, where)


def sas_decode_set_fused(enable: bool) -> None:
    """Process-wide choice of decode implementation: the single persistent launch (True, the
    default, where the shapes allow it) or the three-launch decode (False)."""
    _check(_lib.sas_decode_set_fused(1 if enable else 0), "sas_decode_set_fused")


def decode_noalloc_error_code() -> int:
    """Error word of the last sas_decode_noalloc call on the current device (0 = none). The
    read is ordered after the work queued on the current stream."""
    addr = _vp()
    _check(_lib.sas_decode_noalloc_error_word(ctypes.byref(addr)), "sas_decode_noalloc_error_word")
    out = np.zeros(1, dtype=np.int32)
    torch.cuda.current_stream().synchronize()
    cudart = ctypes.CDLL("libcudart.so.12")          # the runtime torch has already loaded
    cudart.cudaMemcpy.argtypes = [_vp, _vp, _sz, ctypes.c_int]
    err = cudart.cudaMemcpy(out.ctypes.data, addr.value, 4, 2)   # 2 = device to host
    if err != 0:
        raise RuntimeError(f"reading the no-alloc error word failed: cudaError {err}")
    return int(out[0])


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def rope_tables(positions: int, rot_dim: int, base: float = 1e6):
    """Host fp32 cos/sin tables [positions, rot_dim/2] built by the library in double."""
    c = np.empty((positions, rot_dim // 2), dtype=np.float32)
    s = np.empty_like(c)
    _check(_lib.sas_rope_tables(positions, rot_dim, base, c.ctypes.data, s.ctypes.data),
           "sas_rope_tables")
    return c, s


def _dtype_code(dt) -> int:
    if dt == torch.bfloat16:
        return SAS_BF16
    if dt == torch.float32:
        return SAS_FP32
    raise ValueError(f"unsupported dtype {dt}")


@dataclasses.dataclass
class Problem:
    """A packed prefill/training problem plus the device buffers it points at."""
    cu_seqlens: torch.Tensor        # int32 [batch+1], device
    max_seqlen: int
    total_tokens: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block: int
    topk: int
    gate_hidden: int
    dtype: torch.dtype
    rms_eps: float = 1e-6
    gate_rope_base: float = 1e6
    rope_cos: torch.Tensor | None = None
    rope_sin: torch.Tensor | None = None
    gate_heads: int = 0             # 0 / num_kv_heads: one gate per KV group; num_q_heads: per query head

    def __post_init__(self):
        if self.rope_cos is None:
            c, s = rope_tables(self.max_seqlen, self.gate_hidden, self.gate_rope_base)
            dev = self.cu_seqlens.device
            self.rope_cos = torch.from_numpy(c).to(dev)
            self.rope_sin = torch.from_numpy(s).to(dev)
        self._c = SasProblem(len(self.cu_seqlens) - 1, self.total_tokens, self.max_seqlen,
                             self.num_q_heads, self.num_kv_heads, self.head_dim, self.block,
                             self.topk, self.gate_hidden, self.rms_eps, _dtype_code(self.dtype),
                             _ptr(self.cu_seqlens), _ptr(self.rope_cos), _ptr(self.rope_sin),
                             int(self.gate_heads or 0))

    @property
    def sel_heads(self) -> int:
        """gate (selection) heads Hs: the second axis of idx / logg / dlogg / scores"""
        return self.gate_heads or self.num_kv_heads

    @property
    def batch(self) -> int:
        return len(self.cu_seqlens) - 1

    @property
    def max_blocks(self) -> int:
        return (self.max_seqlen + self.block - 1) // self.block

    @property
    def device(self):
        return self.cu_seqlens.device

    @property
    def ref(self):
        return ctypes.byref(self._c)

    @classmethod
    def from_lengths(cls, lengths, device, **kw):
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32,
                          device=device)
        return cls(cu_seqlens=cu, max_seqlen=int(max(lengths)), total_tokens=int(sum(lengths)), **kw)


def sas_pool_keys(p: Problem, k_nope, pooled=None, stream=None):
    if pooled is None:
        pooled = torch.empty((p.batch, p.max_blocks, p.num_kv_heads, 3 * p.head_dim),
                             dtype=torch.float32, device=p.device)
    _check(_lib.sas_pool_keys(p.ref, _ptr(k_nope), _ptr(pooled), _stream(stream)), "sas_pool_keys")
    return pooled


def sas_gate_keys(p: Problem, pooled, wk, knorm_w, gate_keys=None, stream=None):
    if gate_keys is None:
        gate_keys = torch.empty((p.batch, p.max_blocks, p.num_kv_heads, p.gate_hidden),
                                dtype=torch.float32, device=p.device)
    _check(_lib.sas_gate_keys(p.ref, _ptr(pooled), _ptr(wk), _ptr(knorm_w), _ptr(gate_keys),
                              _stream(stream)), "sas_gate_keys")
    return gate_keys


def gate_scores_workspace(p: Problem):
    """A workspace of the size sas_gate_scores asks for."""
    return _workspace(_lib.sas_gate_scores_workspace_size, p.ref, p.device)


def sas_gate_scores(p: Problem, q_nope, k_nope, gate_keys, wq, qnorm_w, wk, knorm_w,
                    scores=None, lse=None, workspace=None, stream=None):
    if scores is None:
        scores = torch.empty((p.total_tokens, p.sel_heads, p.max_blocks), dtype=torch.float32,
                             device=p.device)
    if lse is None:
        lse = torch.empty((p.total_tokens, p.sel_heads), dtype=torch.float32, device=p.device)
    ws = workspace if workspace is not None else gate_scores_workspace(p)
    _check(_lib.sas_gate_scores(p.ref, _ptr(q_nope), _ptr(k_nope), _ptr(gate_keys), _ptr(wq),
                                _ptr(qnorm_w), _ptr(wk), _ptr(knorm_w), _ptr(scores), _ptr(lse),
                                _ptr(ws), ws.numel(), _stream(stream)), "sas_gate_scores")
    return scores, lse


def gate_bwd_workspace(p: Problem):
    """A workspace of the size sas_gate_bwd asks for."""
    return _workspace(_lib.sas_gate_bwd_workspace_size, p.ref, p.device)


def sas_gate_bwd(p: Problem, q_nope, k_nope, pooled, wq, qnorm_w, wk, knorm_w, idx, dlogg,
                 workspace=None, stream=None):
    """Router backward: (dwq, dqnorm_w, dwk, dknorm_w), fp32, through the kept log-gates."""
    G, h, d, Hkv = p.num_q_heads // p.num_kv_heads, p.gate_hidden, p.head_dim, p.num_kv_heads
    dwq = torch.empty((Hkv, h, G * d), dtype=torch.float32, device=p.device)
    dwk = torch.empty((Hkv, h, 3 * d), dtype=torch.float32, device=p.device)
    dqn = torch.empty((h,), dtype=torch.float32, device=p.device)
    dkn = torch.empty((h,), dtype=torch.float32, device=p.device)
    ws = workspace if workspace is not None else gate_bwd_workspace(p)
    _check(_lib.sas_gate_bwd(p.ref, _ptr(q_nope), _ptr(k_nope), _ptr(pooled), _ptr(wq),
                             _ptr(qnorm_w), _ptr(wk), _ptr(knorm_w), _ptr(idx), _ptr(dlogg),
                             _ptr(dwq), _ptr(dqn), _ptr(dwk), _ptr(dkn), _ptr(ws), ws.numel(),
                             _stream(stream)), "sas_gate_bwd")
    return dwq, dqn, dwk, dkn


def sas_topk(p: Problem, scores, lse, idx=None, logg=None, stream=None):
    shape = (p.total_tokens, p.sel_heads, p.topk + 1)
    if idx is None:
        idx = torch.empty(shape, dtype=torch.int32, device=p.device)
    if logg is None:
        logg = torch.empty(shape, dtype=torch.float32, device=p.device)
    _check(_lib.sas_topk(p.ref, _ptr(scores), _ptr(lse), _ptr(idx), _ptr(logg), _stream(stream)),
           "sas_topk")
    return idx, logg


def _workspace(fn, prob_ref, device):
    """A fresh workspace of the size the library asks for (torch's stream-ordered allocator)."""
    n = _sz(0)
    _check(fn(prob_ref, ctypes.byref(n)), fn.__name__)
    return torch.zeros(max(int(n.value), 256), dtype=torch.uint8, device=device)


def attn_fwd_workspace(p: Problem):
    """A zeroed workspace of the size sas_attn_fwd asks for (word 0: pipeline error code)."""
    return _workspace(_lib.sas_attn_fwd_workspace_size, p.ref, p.device)


def attn_bwd_workspace(p: Problem):
    """A zeroed workspace of the size sas_attn_bwd asks for."""
    return _workspace(_lib.sas_attn_bwd_workspace_size, p.ref, p.device)


def sas_attn_fwd(p: Problem, q, k, v, idx, logg, o=None, lse=None, workspace=None, stream=None,
                 check: bool = False):
    """Gated sparse attention forward. check=True waits for the call and raises
    SasDeviceError if its workspace error word is set."""
    if o is None:
        o = torch.empty((p.total_tokens, p.num_q_heads, p.head_dim), dtype=p.dtype, device=p.device)
    if lse is None:
        lse = torch.empty((p.total_tokens, p.num_q_heads), dtype=torch.float32, device=p.device)
    ws = workspace if workspace is not None else _workspace(_lib.sas_attn_fwd_workspace_size, p.ref, p.device)
    _check(_lib.sas_attn_fwd(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(logg), _ptr(o),
                             _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "sas_attn_fwd")
    if check:
        check_workspace(ws, "sas_attn_fwd")
    return o, lse


def sas_attn_bwd(p: Problem, q, k, v, o, dout, lse, idx, logg, dq=None, dk=None, dv=None,
                 dlogg=None, workspace=None, stream=None, check: bool = False):
    """Backward of the gated sparse attention; check=True as in sas_attn_fwd."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if dlogg is None:
        dlogg = torch.empty((p.total_tokens, p.sel_heads, p.topk + 1), dtype=torch.float32,
                            device=p.device)
    ws = workspace if workspace is not None else _workspace(_lib.sas_attn_bwd_workspace_size, p.ref, p.device)
    _check(_lib.sas_attn_bwd(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                             _ptr(idx), _ptr(logg), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlogg),
                             _ptr(ws), ws.numel(), _stream(stream)), "sas_attn_bwd")
    if check:
        check_workspace(ws, "sas_attn_bwd")
    return dq, dk, dv, dlogg


def gate_select_workspace(p: Problem):
    """A workspace of the size sas_gate_select asks for."""
    return _workspace(_lib.sas_gate_select_workspace_size, p.ref, p.device)


def sas_gate_select(p: Problem, q_nope, k_nope, gate_keys, wq, qnorm_w, wk, knorm_w, idx=None,
                    logg=None, lse=None, workspace=None, stream=None, want_lse: bool = False):
    """Gate scores + Top-K in one pass (scores never written for the fused shapes).
    Returns (idx, logg), or (idx, logg, lse) with want_lse."""
    shape = (p.total_tokens, p.sel_heads, p.topk + 1)
    if idx is None:
        idx = torch.empty(shape, dtype=torch.int32, device=p.device)
    if logg is None:
        logg = torch.empty(shape, dtype=torch.float32, device=p.device)
    if want_lse and lse is None:
        lse = torch.empty((p.total_tokens, p.sel_heads), dtype=torch.float32, device=p.device)
    ws = workspace if workspace is not None else gate_select_workspace(p)
    _check(_lib.sas_gate_select(p.ref, _ptr(q_nope), _ptr(k_nope), _ptr(gate_keys), _ptr(wq),
                                _ptr(qnorm_w), _ptr(wk), _ptr(knorm_w), _ptr(idx), _ptr(logg),
                                _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "sas_gate_select")
    return (idx, logg, lse) if want_lse else (idx, logg)


def prefill_selection(p: Problem, q_nope, k_nope, wq, qnorm_w, wk, knorm_w, stream=None,
                      fused: bool = True):
    """A1..A4 in order: pool -> gate keys -> scores + Top-K (one fused pass, or the separate
    score and Top-K calls with fused=False). Returns (idx, logg)."""
    pooled = sas_pool_keys(p, k_nope, stream=stream)
    gk = sas_gate_keys(p, pooled, wk, knorm_w, stream=stream)
    if fused:
        return sas_gate_select(p, q_nope, k_nope, gk, wq, qnorm_w, wk, knorm_w, stream=stream)
    scores, lse = sas_gate_scores(p, q_nope, k_nope, gk, wq, qnorm_w, wk, knorm_w, stream=stream)
    return sas_topk(p, scores, lse, stream=stream)


@dataclasses.dataclass
class DecodeProblem:
    seqlens: torch.Tensor           # int32 [batch], device
    capacity: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block: int
    topk: int
    gate_hidden: int
    dtype: torch.dtype
    rms_eps: float = 1e-6
    gate_rope_base: float = 1e6
    rope_cos: torch.Tensor | None = None
    rope_sin: torch.Tensor | None = None
    gated: bool = True              # False: hard selection, no log-gate in the attention logits
    gate_heads: int = 0             # 0 / num_kv_heads: one gate per KV group; num_q_heads: per query head

    def __post_init__(self):
        if self.rope_cos is None:
            c, s = rope_tables(self.capacity, self.gate_hidden, self.gate_rope_base)
            dev = self.seqlens.device
            self.rope_cos = torch.from_numpy(c).to(dev)
            self.rope_sin = torch.from_numpy(s).to(dev)
        self._c = SasDecodeProblem(len(self.seqlens), self.capacity, self.num_q_heads,
                                   self.num_kv_heads, self.head_dim, self.block, self.topk,
                                   self.gate_hidden, self.rms_eps, _dtype_code(self.dtype),
                                   _ptr(self.seqlens), _ptr(self.rope_cos), _ptr(self.rope_sin),
                                   0 if self.gated else 1, int(self.gate_heads or 0))

    @property
    def sel_heads(self) -> int:
        return self.gate_heads or self.num_kv_heads

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def device(self):
        return self.seqlens.device

    @property
    def ref(self):
        return ctypes.byref(self._c)


def sas_decode(p: DecodeProblem, q, q_nope, k_cache, v_cache, gate_key_cache, cur_pool, wq,
               qnorm_w, wk, knorm_w, o=None, idx_out=None, logg_out=None, workspace=None,
               stream=None, want_selection: bool = False, check: bool = False):
    """One sparse decode step; check=True waits for the call and raises SasDeviceError if
    its workspace error word is set."""
    if o is None:
        o = torch.empty((p.batch, p.num_q_heads, p.head_dim), dtype=p.dtype, device=p.device)
    if want_selection and idx_out is None:
        idx_out = torch.empty((p.batch, p.sel_heads, p.topk + 1), dtype=torch.int32,
                              device=p.device)
        logg_out = torch.empty((p.batch, p.sel_heads, p.topk + 1), dtype=torch.float32,
                               device=p.device)
    ws = workspace if workspace is not None else _workspace(_lib.sas_decode_workspace_size, p.ref, p.device)
    _check(_lib.sas_decode(p.ref, _ptr(q), _ptr(q_nope), _ptr(k_cache), _ptr(v_cache),
                           _ptr(gate_key_cache), _ptr(cur_pool), _ptr(wq), _ptr(qnorm_w), _ptr(wk),
                           _ptr(knorm_w), _ptr(o), _ptr(idx_out), _ptr(logg_out), _ptr(ws),
                           ws.numel(), _stream(stream)), "sas_decode")
    if check:
        check_workspace(ws, "sas_decode")
    return (o, idx_out, logg_out) if want_selection else o


def sas_decode_paged(p: DecodeProblem, page_table, num_pages: int, q, q_nope, k_pages, v_pages,
                     gate_key_pages, cur_pool, wq, qnorm_w, wk, knorm_w, o=None, idx_out=None,
                     logg_out=None, workspace=None, stream=None, want_selection: bool = False,
                     check: bool = False):
    """One sparse decode step over paged caches: page_table int32 [batch, ceil(capacity/B)],
    k_pages / v_pages [num_pages, Hkv, B, d], gate_key_pages bf16 [num_pages, Hkv, h]."""
    if o is None:
        o = torch.empty((p.batch, p.num_q_heads, p.head_dim), dtype=p.dtype, device=p.device)
    if want_selection and idx_out is None:
        idx_out = torch.empty((p.batch, p.sel_heads, p.topk + 1), dtype=torch.int32,
                              device=p.device)
        logg_out = torch.empty((p.batch, p.sel_heads, p.topk + 1), dtype=torch.float32,
                               device=p.device)
    ws = workspace if workspace is not None else _workspace(_lib.sas_decode_workspace_size, p.ref, p.device)
    _check(_lib.sas_decode_paged(p.ref, _ptr(page_table), int(num_pages), _ptr(q), _ptr(q_nope),
                                 _ptr(k_pages), _ptr(v_pages), _ptr(gate_key_pages), _ptr(cur_pool),
                                 _ptr(wq), _ptr(qnorm_w), _ptr(wk), _ptr(knorm_w), _ptr(o),
                                 _ptr(idx_out), _ptr(logg_out), _ptr(ws), ws.numel(),
                                 _stream(stream)), "sas_decode_paged")
    if check:
        check_workspace(ws, "sas_decode_paged")
    return (o, idx_out, logg_out) if want_selection else o


def lib_handle():
    return _lib


def kernel_launches() -> int:
    """Kernels the library has launched from this thread so far."""
    return int(_lib.sas_kernel_launches())
