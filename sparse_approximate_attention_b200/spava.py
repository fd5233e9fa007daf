"""Python binding of libspava (the C ABI in include/spava.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels
of libspava.so.  PyTorch supplies device memory and the current stream.  The
library must have been built (``python -m sparse_approximate_attention_b200.build``);
without it every call raises -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspava.so")

SCORE_KINDS = {"linear": 0, "softmax": 1, "context": 2}   # SPAVA_SCORE_*
STATUS = {0: "SPAVA_OK", 1: "SPAVA_ERR_INVALID_ARG", 2: "SPAVA_ERR_UNSUPPORTED",
          3: "SPAVA_ERR_WORKSPACE", 4: "SPAVA_ERR_CUDA", 5: "SPAVA_ERR_DEVICE"}


class SpavaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class _Problem(ctypes.Structure):
    _fields_ = [("num_hosts", ctypes.c_int32), ("anchor_len", ctypes.c_int32),
                ("block_lens", ctypes.POINTER(ctypes.c_int32)), ("query_len", ctypes.c_int32),
                ("lp", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("score_kind", ctypes.c_int32),
                ("host_mask", ctypes.c_uint32)]


class _Sizes(ctypes.Structure):
    _fields_ = [("seq_len", ctypes.c_int64), ("query_start", ctypes.c_int64),
                ("score_cols", ctypes.c_int64), ("passing_rows", ctypes.c_int64),
                ("attn_pairs", ctypes.c_int64), ("attn_flops", ctypes.c_double),
                ("attn_tiles", ctypes.c_int64), ("workspace_bytes", ctypes.c_size_t)]


_lib = None
_VP = ctypes.c_void_p
_PP = ctypes.POINTER(_Problem)
_SIGS = {
    "spava_problem_sizes": [_PP, ctypes.POINTER(_Sizes)],
    "spava_workspace_size": [_PP, ctypes.POINTER(ctypes.c_size_t)],
    "spava_score": [_PP, _VP, _VP, _VP, _VP, _VP],
    "spava_score_variant": [_PP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP],
    "spava_select_topk": [_PP, _VP, _VP, _VP],
    "spava_gather_passing": [_PP, _VP, _VP, _VP, _VP, _VP, _VP],
    "spava_compress": [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "spava_attn_fwd": [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "spava_lse_merge": [_PP, _VP, _VP, _VP, _VP, _VP],
    "spava_layer_fwd": [_PP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP],
    "spava_device_error": [ctypes.POINTER(ctypes.c_uint32)],
    "spava_layer_fwd_noalloc": [_PP, _VP, _VP, _VP, _VP, _VP, _VP],
    "spava_debug_wait_timeout": [_VP, ctypes.c_uint64, _VP],
    "spava_debug_attn_abort": [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int32, ctypes.c_uint64, _VP],
}


def lib() -> ctypes.CDLL:
    """Load libspava.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_approximate_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.spava_status_string.argtypes = [ctypes.c_int]
        L.spava_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise SpavaError(fn, code)


class Problem:
    """One layer's problem: H physical hosts (2H context blocks), anchor
    length la, context block lengths, query length lq, passing length lp,
    query/KV heads and head_dim.  host_mask (0 = all) selects the virtual
    hosts a call computes (bit h: host h; the anchor rows go with bit 0)."""

    def __init__(self, num_hosts: int, anchor_len: int, block_lens: Sequence[int],
                 query_len: int, lp: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, softmax_scale: float = 0.0, score_kind: str = "linear",
                 host_mask: int = 0):
        self.num_hosts, self.anchor_len = int(num_hosts), int(anchor_len)
        self.block_lens = [int(x) for x in block_lens]
        self.query_len, self.lp = int(query_len), int(lp)
        self.num_q_heads, self.num_kv_heads = int(num_q_heads), int(num_kv_heads)
        self.head_dim, self.softmax_scale = int(head_dim), float(softmax_scale)
        self.score_kind = score_kind
        self.host_mask = int(host_mask)
        self._arr = (ctypes.c_int32 * max(1, len(self.block_lens)))(*self.block_lens)
        self._c = _Problem(self.num_hosts, self.anchor_len, self._arr, self.query_len, self.lp,
                           self.num_q_heads, self.num_kv_heads, self.head_dim, self.softmax_scale,
                           SCORE_KINDS[score_kind], self.host_mask)

    @classmethod
    def from_workload(cls, wl, score_kind: str = "linear", host_mask: int = 0) -> "Problem":
        return cls(wl.num_hosts, wl.anchor_len, wl.block_lens, wl.query_len, wl.lp,
                   wl.num_q_heads, wl.num_kv_heads, wl.head_dim, score_kind=score_kind,
                   host_mask=host_mask)

    def with_hosts(self, host_mask: int) -> "Problem":
        """The same problem restricted to the virtual hosts of host_mask."""
        return Problem(self.num_hosts, self.anchor_len, self.block_lens, self.query_len, self.lp,
                       self.num_q_heads, self.num_kv_heads, self.head_dim, self.softmax_scale,
                       self.score_kind, host_mask)

    @property
    def ref(self):
        return ctypes.byref(self._c)

    def sizes(self) -> dict:
        s = _Sizes()
        _check("spava_problem_sizes", lib().spava_problem_sizes(self.ref, ctypes.byref(s)))
        return {k: getattr(s, k) for k, _ in _Sizes._fields_}

    @property
    def V(self) -> int:
        return 2 * self.num_hosts


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def _shapes(p: Problem):
    sz = p.sizes()
    n, hq, hkv, d, V = sz["seq_len"], p.num_q_heads, p.num_kv_heads, p.head_dim, p.V
    return sz, dict(Q=(n, hq, d), K=(n, hkv, d), V=(n, hkv, d), O=(n, hq, d), lse=(hq, n),
                    qsum=(hkv, d), scores=(hkv, sz["score_cols"]), idx=(V - 1, hkv, p.lp),
                    Kp=(sz["passing_rows"], hkv, d), O_part=(V, p.query_len, hq, d),
                    lse_part=(V, hq, p.query_len))


def score(p: Problem, Q, K, qsum=None, scores=None, stream=None):
    sz, sh = _shapes(p)
    _need(Q, torch.bfloat16, sh["Q"], "Q")
    _need(K, torch.bfloat16, sh["K"], "K")
    qsum = torch.empty(sh["qsum"], dtype=torch.float32, device=Q.device) if qsum is None else qsum
    scores = torch.empty(sh["scores"], dtype=torch.float32, device=Q.device) if scores is None else scores
    _need(qsum, torch.float32, sh["qsum"], "qsum")
    _need(scores, torch.float32, sh["scores"], "scores")
    _check("spava_score", lib().spava_score(p.ref, _ptr(Q), _ptr(K), _ptr(qsum), _ptr(scores), _stream(stream)))
    return qsum, scores


def score_variant(p: Problem, Q, K, scores=None, workspace=None, stream=None):
    """Step 1 under the problem's selector (p.score_kind), into scores [Hkv, S]."""
    sz, sh = _shapes(p)
    _need(Q, torch.bfloat16, sh["Q"], "Q")
    _need(K, torch.bfloat16, sh["K"], "K")
    scores = torch.empty(sh["scores"], dtype=torch.float32, device=Q.device) if scores is None else scores
    _need(scores, torch.float32, sh["scores"], "scores")
    if workspace is None:
        workspace = torch.empty(max(1, sz["workspace_bytes"]), dtype=torch.uint8, device=Q.device)
    _check("spava_score_variant", lib().spava_score_variant(
        p.ref, _ptr(Q), _ptr(K), _ptr(scores), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return scores


def select_topk(p: Problem, scores, idx=None, stream=None):
    sz, sh = _shapes(p)
    _need(scores, torch.float32, sh["scores"], "scores")
    idx = torch.empty(sh["idx"], dtype=torch.int32, device=scores.device) if idx is None else idx
    _need(idx, torch.int32, sh["idx"], "idx")
    _check("spava_select_topk", lib().spava_select_topk(p.ref, _ptr(scores), _ptr(idx), _stream(stream)))
    return idx


def gather_passing(p: Problem, K, V, idx, Kp=None, Vp=None, stream=None):
    sz, sh = _shapes(p)
    _need(K, torch.bfloat16, sh["K"], "K")
    _need(V, torch.bfloat16, sh["V"], "V")
    _need(idx, torch.int32, sh["idx"], "idx")
    Kp = torch.empty(sh["Kp"], dtype=torch.bfloat16, device=K.device) if Kp is None else Kp
    Vp = torch.empty(sh["Kp"], dtype=torch.bfloat16, device=K.device) if Vp is None else Vp
    _need(Kp, torch.bfloat16, sh["Kp"], "Kp")
    _need(Vp, torch.bfloat16, sh["Kp"], "Vp")
    _check("spava_gather_passing", lib().spava_gather_passing(
        p.ref, _ptr(K), _ptr(V), _ptr(idx), _ptr(Kp), _ptr(Vp), _stream(stream)))
    return Kp, Vp


def compress(p: Problem, Q, K, V, qsum=None, scores=None, idx=None, Kp=None, Vp=None, stream=None):
    """Steps 1-3 fused (query sum, then scores, top-lp indices and passing
    buffer in one cluster launch)."""
    sz, sh = _shapes(p)
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, sh[nm], nm)
    dev = Q.device
    qsum = torch.empty(sh["qsum"], dtype=torch.float32, device=dev) if qsum is None else qsum
    scores = torch.empty(sh["scores"], dtype=torch.float32, device=dev) if scores is None else scores
    idx = torch.empty(sh["idx"], dtype=torch.int32, device=dev) if idx is None else idx
    Kp = torch.empty(sh["Kp"], dtype=torch.bfloat16, device=dev) if Kp is None else Kp
    Vp = torch.empty(sh["Kp"], dtype=torch.bfloat16, device=dev) if Vp is None else Vp
    for t, nm, dt, k in ((qsum, "qsum", torch.float32, "qsum"), (scores, "scores", torch.float32, "scores"),
                         (idx, "idx", torch.int32, "idx"), (Kp, "Kp", torch.bfloat16, "Kp"),
                         (Vp, "Vp", torch.bfloat16, "Kp")):
        _need(t, dt, sh[k], nm)
    _check("spava_compress", lib().spava_compress(
        p.ref, _ptr(Q), _ptr(K), _ptr(V), _ptr(qsum), _ptr(scores), _ptr(idx), _ptr(Kp), _ptr(Vp),
        _stream(stream)))
    return qsum, scores, idx, Kp, Vp


def attn_fwd(p: Problem, Q, K, V, Kp, Vp, O=None, lse=None, O_part=None, lse_part=None, stream=None):
    sz, sh = _shapes(p)
    dev = Q.device
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, sh[nm], nm)
    if sz["passing_rows"] > 0:
        _need(Kp, torch.bfloat16, sh["Kp"], "Kp")
        _need(Vp, torch.bfloat16, sh["Kp"], "Vp")
    O = torch.empty(sh["O"], dtype=torch.bfloat16, device=dev) if O is None else O
    lse = torch.empty(sh["lse"], dtype=torch.float32, device=dev) if lse is None else lse
    O_part = torch.empty(sh["O_part"], dtype=torch.float32, device=dev) if O_part is None else O_part
    lse_part = torch.empty(sh["lse_part"], dtype=torch.float32, device=dev) if lse_part is None else lse_part
    _need(O, torch.bfloat16, sh["O"], "O")
    _need(lse, torch.float32, sh["lse"], "lse")
    _need(O_part, torch.float32, sh["O_part"], "O_part")
    _need(lse_part, torch.float32, sh["lse_part"], "lse_part")
    _check("spava_attn_fwd", lib().spava_attn_fwd(
        p.ref, _ptr(Q), _ptr(K), _ptr(V), _ptr(Kp), _ptr(Vp), _ptr(O), _ptr(lse), _ptr(O_part),
        _ptr(lse_part), _stream(stream)))
    return O, lse, O_part, lse_part


def lse_merge(p: Problem, O_part, lse_part, O, lse, stream=None):
    sz, sh = _shapes(p)
    _need(O_part, torch.float32, sh["O_part"], "O_part")
    _need(lse_part, torch.float32, sh["lse_part"], "lse_part")
    _need(O, torch.bfloat16, sh["O"], "O")
    _need(lse, torch.float32, sh["lse"], "lse")
    _check("spava_lse_merge", lib().spava_lse_merge(
        p.ref, _ptr(O_part), _ptr(lse_part), _ptr(O), _ptr(lse), _stream(stream)))
    return O, lse


def workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t()
    _check("spava_workspace_size", lib().spava_workspace_size(p.ref, ctypes.byref(n)))
    return n.value


def layer_fwd(p: Problem, Q, K, V, O=None, lse=None, workspace=None, stream=None):
    """The whole layer (score -> top-lp -> gather -> attention -> merge)."""
    sz, sh = _shapes(p)
    dev = Q.device
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, sh[nm], nm)
    O = torch.empty(sh["O"], dtype=torch.bfloat16, device=dev) if O is None else O
    lse = torch.empty(sh["lse"], dtype=torch.float32, device=dev) if lse is None else lse
    _need(O, torch.bfloat16, sh["O"], "O")
    _need(lse, torch.float32, sh["lse"], "lse")
    if workspace is None:
        workspace = torch.empty(max(1, sz["workspace_bytes"]), dtype=torch.uint8, device=dev)
    _check("spava_layer_fwd", lib().spava_layer_fwd(
        p.ref, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return O, lse


def device_error() -> int:
    """Device-side error word (synchronizes; clears it)."""
    v = ctypes.c_uint32()
    _check("spava_device_error", lib().spava_device_error(ctypes.byref(v)))
    return v.value


def layer_fwd_noalloc(p: Problem, Q, K, V, O, lse, stream=None):
    """The whole layer without a workspace, for callers that cannot allocate
    device memory: its intermediates live in a fixed 64 MiB array inside the
    library (problems whose workspace is larger are rejected).  O and lse are
    caller-provided.  Calls that overlap on the GPU race on that array."""
    sz, sh = _shapes(p)
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O")):
        _need(t, torch.bfloat16, sh[nm], nm)
    _need(lse, torch.float32, sh["lse"], "lse")
    _check("spava_layer_fwd_noalloc", lib().spava_layer_fwd_noalloc(
        p.ref, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _stream(stream)))
    return O, lse


def debug_wait_timeout(limit_ns: int, stream=None):
    """Test hook: a bounded mbarrier wait that runs out after limit_ns.
    Returns (wait result, abort flag, drain result, elapsed ns)."""
    out = torch.zeros(4, dtype=torch.int64, device="cuda")
    _check("spava_debug_wait_timeout", lib().spava_debug_wait_timeout(_ptr(out), int(limit_ns), _stream(stream)))
    return tuple(int(v) for v in out.cpu().tolist())


def debug_attn_abort(p: Problem, Q, K, V, Kp, Vp, skip_k_tile: int, limit_ns: int, stream=None):
    """Test hook: the attention launch with key tile skip_k_tile left
    unloaded and every wait limited to limit_ns (its outputs are invalid)."""
    sh = _shapes(p)[1]
    dev = Q.device
    O = torch.empty(sh["O"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(sh["lse"], dtype=torch.float32, device=dev)
    O_part = torch.empty(sh["O_part"], dtype=torch.float32, device=dev)
    lse_part = torch.empty(sh["lse_part"], dtype=torch.float32, device=dev)
    _check("spava_debug_attn_abort", lib().spava_debug_attn_abort(
        p.ref, _ptr(Q), _ptr(K), _ptr(V), _ptr(Kp), _ptr(Vp), _ptr(O), _ptr(lse), _ptr(O_part), _ptr(lse_part),
        int(skip_k_tile), int(limit_ns), _stream(stream)))
