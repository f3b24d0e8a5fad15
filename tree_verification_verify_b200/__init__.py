"""B200-native tree verification: Python binding of libtreeverify.so.

Argument marshalling only.  Every step of the path runs in the library's
CUDA kernels (include/tree_verify.h); PyTorch supplies device memory and the
current stream.  There is no CPU fallback: without the built library or a
CUDA device these functions raise.

    tree_verify_attn   tree-masked attention over prefix + ancestors
    tree_accept        acceptance walk (greedy / speculative sampling /
                       deterministic-tree sampling)
    tree_expand_init / tree_expand_topb
                       batched best-first expansion rounds
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = ["lib", "version", "status_string", "tree_verify_attn", "tree_verify_attn_merge", "tree_accept", "tree_accept_noalloc",
           "tree_expand_init", "tree_expand_topb", "ExpandState", "EXPAND_MODES", "tree_commit_kv", "philox_uniforms",
           "TVError", "MODES"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtreeverify.so")

c_i32, c_i64, c_u64, c_f32, c_vp, c_size = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                             ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t)

TV_FP32, TV_BF16 = 0, 1
MODES = {"auto": 0, "greedy": 1, "specsample": 2, "specexec": 3}


class AttnArgs(ctypes.Structure):
    _fields_ = [("dtype", c_i32), ("B", c_i32), ("T", c_i32), ("Hq", c_i32), ("Hkv", c_i32),
                ("d", c_i32), ("Lmax", c_i32),
                ("q", c_vp), ("q_sb", c_i64), ("q_st", c_i64), ("q_sh", c_i64),
                ("k_cache", c_vp), ("v_cache", c_vp), ("kv_sb", c_i64), ("kv_sl", c_i64), ("kv_sh", c_i64),
                ("prefix_len", c_vp),
                ("k_tree", c_vp), ("v_tree", c_vp), ("kt_sb", c_i64), ("kt_st", c_i64), ("kt_sh", c_i64),
                ("parent", c_vp), ("parent_sb", c_i64),
                ("n_nodes", c_vp),
                ("scale", c_f32), ("sparse_topk", c_i32), ("block_size", c_i32),
                ("k_block_mean", c_vp),
                ("out", c_vp), ("o_sb", c_i64), ("o_st", c_i64), ("o_sh", c_i64),
                ("lse", c_vp), ("sel_blocks", c_vp), ("dev_status", c_vp), ("prefix_only", c_i32)]


class AttnMergeArgs(ctypes.Structure):
    _fields_ = [("dtype", c_i32), ("N", c_i32), ("B", c_i32), ("T", c_i32), ("Hq", c_i32), ("d", c_i32),
                ("o_parts", c_vp), ("lse_parts", c_vp), ("out", c_vp), ("lse", c_vp)]


class AcceptArgs(ctypes.Structure):
    _fields_ = [("B", c_i32), ("T", c_i32), ("V", c_i32),
                ("target_logits", c_vp), ("tl_sb", c_i64), ("tl_st", c_i64),
                ("draft_probs", c_vp), ("dp_sb", c_i64), ("dp_st", c_i64),
                ("draft_tokens", c_vp), ("tok_sb", c_i64),
                ("parent", c_vp), ("parent_sb", c_i64),
                ("n_nodes", c_vp),
                ("mode", c_i32), ("temperature", c_f32), ("seed", c_u64), ("step", c_u64),
                ("n_accepted", c_vp), ("accepted_nodes", c_vp), ("out_tokens", c_vp),
                ("min_margin", c_vp), ("dev_status", c_vp)]


class ExpandArgs(ctypes.Structure):
    _fields_ = [("V", c_i32), ("R", c_i32), ("Bsel", c_i32), ("budget", c_i32),
                ("draft_temperature", c_f32),
                ("draft_logits", c_vp), ("ld_logits", c_i64),
                ("row_node", c_vp),
                ("n_nodes", c_vp), ("parent", c_vp), ("token", c_vp), ("logp", c_vp),
                ("pool", c_vp), ("pool_bytes", c_size),
                ("frontier", c_vp), ("n_appended", c_vp), ("dev_status", c_vp), ("mode", c_i32)]


EXPAND_MODES = {"bestfirst": 0, "beam": 1}


class CommitArgs(ctypes.Structure):
    _fields_ = [("dtype", c_i32), ("B", c_i32), ("T", c_i32), ("Hkv", c_i32), ("d", c_i32), ("Lmax", c_i32),
                ("k_cache", c_vp), ("v_cache", c_vp), ("kv_sb", c_i64), ("kv_sl", c_i64), ("kv_sh", c_i64),
                ("prefix_len", c_vp),
                ("k_tree", c_vp), ("v_tree", c_vp), ("kt_sb", c_i64), ("kt_st", c_i64), ("kt_sh", c_i64),
                ("n_accepted", c_vp), ("accepted_nodes", c_vp), ("acc_sb", c_i64),
                ("dev_status", c_vp)]


class TVError(RuntimeError):
    pass


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise TVError(f"{LIB_PATH} is missing: build it with "
                          "`python -m tree_verification_verify_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in (("tree_verify_attn", [ctypes.POINTER(AttnArgs), c_vp, c_size, c_vp]),
                           ("tree_verify_attn_merge", [ctypes.POINTER(AttnMergeArgs), c_vp]),
                           ("tree_accept", [ctypes.POINTER(AcceptArgs), c_vp, c_size, c_vp]),
                           ("tree_accept_noalloc", [ctypes.POINTER(AcceptArgs), c_vp]),
                           ("tree_expand_topb", [ctypes.POINTER(ExpandArgs), c_vp, c_size, c_vp]),
                           ("tree_expand_init", [ctypes.POINTER(ExpandArgs), c_i32, c_vp]),
                           ("tree_commit_kv", [ctypes.POINTER(CommitArgs), c_vp]),
                           ("tv_philox_uniforms", [c_u64, c_u64, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp]),
                           ("tv_expand_exp", [c_vp, c_vp, c_i32, c_vp]),
                           ("tv_expand_set_wait_limit", [ctypes.c_uint32])):
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        for name, t in (("tree_verify_attn_workspace_size", AttnArgs),
                        ("tree_accept_workspace_size", AcceptArgs),
                        ("tree_expand_workspace_size", ExpandArgs)):
            f = getattr(L, name)
            f.argtypes = [ctypes.POINTER(t)]
            f.restype = c_size
        L.tv_attn_path.argtypes = [ctypes.POINTER(AttnArgs)]
        L.tv_attn_path.restype = c_i32
        L.tv_attn_launches.argtypes = [ctypes.POINTER(AttnArgs)]
        L.tv_attn_launches.restype = c_i32
        L.tree_expand_pool_bytes.argtypes = [c_i32, c_i32]
        L.tree_expand_pool_bytes.restype = c_size
        L.tree_verify_version.restype = ctypes.c_char_p
        L.tv_status_string.argtypes = [ctypes.c_int]
        L.tv_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def version() -> str:
    return lib().tree_verify_version().decode()


def status_string(code: int) -> str:
    return lib().tv_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != 0:
        raise TVError(f"{what}: {status_string(code)} (status {code})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need_cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise TVError("tensors must live on a CUDA device (there is no CPU path)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise TVError("tensors must share one device")
    return dev


def _i32(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if t.dtype != torch.int32 or not t.is_contiguous():
        raise TVError("index tensors must be contiguous int32")
    return t


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# Workspaces are zero-filled at allocation and left ready by every call;
# one per (device, stream) so that calls on different streams never share.
_ws_cache = {}


def _workspace(device, stream_handle: int, nbytes: int) -> torch.Tensor:
    key = (device.index, stream_handle)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 256) + 256, dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def _aligned_ptr(buf: torch.Tensor) -> int:
    p = buf.data_ptr()
    return (p + 255) & ~255


# --------------------------------------------------------------- attention

def tree_verify_attn(q, k_cache, v_cache, prefix_len, k_tree, v_tree, parent, n_nodes=None,
                     scale: float = 0.0, sparse_topk: int = 0, block_size: int = 64,
                     k_block_mean=None, out=None, lse=None, want_lse: bool = True,
                     sel_blocks=None, want_sel: bool = False, dev_status=None, stream=None,
                     prefix_only: bool = False):
    """Tree-masked attention (include/tree_verify.h, tree_verify_attn).
    Shapes: q [B][T][Hq][d], caches [B][Lmax][Hkv][d], tree K/V [B][T][Hkv][d]
    (innermost dim contiguous, K and V with equal strides), prefix_len [B],
    parent [B][T], n_nodes [B] or None.  prefix_only: the partial over the
    prefix keys alone (a rank's slice of a split prefix).  Returns
    (out, lse, sel_blocks)."""
    dev = _need_cuda(q, k_cache, v_cache, prefix_len, k_tree, v_tree, parent, n_nodes, k_block_mean)
    if q.dtype == torch.bfloat16:
        dt = TV_BF16
    elif q.dtype == torch.float32:
        dt = TV_FP32
    else:
        raise TVError("q must be bf16 or fp32")
    for t in (k_cache, v_cache, k_tree, v_tree):
        if t.dtype != q.dtype or t.stride(-1) != 1:
            raise TVError("K/V must share q's dtype with a contiguous last dimension")
    if k_cache.stride() != v_cache.stride() or k_tree.stride() != v_tree.stride():
        raise TVError("K and V tensors must have equal strides")
    B, T, Hq, d = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    if q.stride(-1) != 1:
        raise TVError("q must have a contiguous last dimension")
    prefix_len = _i32(prefix_len)
    n_nodes = _i32(n_nodes)
    if parent.dtype != torch.int32 or parent.stride(-1) != 1:
        raise TVError("parent must be int32 with contiguous rows")
    if out is None:
        out = torch.empty(B, T, Hq, d, dtype=q.dtype, device=dev)
    if lse is None and want_lse:
        lse = torch.empty(B, T, Hq, dtype=torch.float32, device=dev)
    if sel_blocks is None and want_sel and sparse_topk > 0:
        sel_blocks = torch.full((B, T, Hkv, sparse_topk), -1, dtype=torch.int32, device=dev)
    if k_block_mean is not None and (k_block_mean.dtype != torch.float32 or not k_block_mean.is_contiguous()):
        raise TVError("k_block_mean must be contiguous fp32")
    a = AttnArgs(dt, B, T, Hq, Hkv, d, Lmax,
                 q.data_ptr(), q.stride(0), q.stride(1), q.stride(2),
                 k_cache.data_ptr(), v_cache.data_ptr(), k_cache.stride(0), k_cache.stride(1), k_cache.stride(2),
                 prefix_len.data_ptr(),
                 k_tree.data_ptr(), v_tree.data_ptr(), k_tree.stride(0), k_tree.stride(1), k_tree.stride(2),
                 parent.data_ptr(), parent.stride(0),
                 _ptr(n_nodes), float(scale), int(sparse_topk), int(block_size), _ptr(k_block_mean),
                 out.data_ptr(), out.stride(0), out.stride(1), out.stride(2),
                 _ptr(lse), _ptr(sel_blocks), _ptr(dev_status), int(bool(prefix_only)))
    L = lib()
    global last_attn_path, last_attn_launches
    last_attn_path = L.tv_attn_path(ctypes.byref(a))
    last_attn_launches = L.tv_attn_launches(ctypes.byref(a))
    need = L.tree_verify_attn_workspace_size(ctypes.byref(a))
    sh = _stream(stream)
    ws = _workspace(dev, sh, need)
    _check(L.tree_verify_attn(ctypes.byref(a), _aligned_ptr(ws), need, sh), "tree_verify_attn")
    return out, lse, sel_blocks


def tree_verify_attn_merge(o_parts, lse_parts, out=None, lse=None, stream=None):
    """Log-sum-exp merge of N attention partials over disjoint key sets
    (include/tree_verify.h, tree_verify_attn_merge): o_parts [N][B][T][Hq][d]
    bf16/fp32, lse_parts [N][B][T][Hq] fp32, both contiguous.  Returns
    (out [B][T][Hq][d], lse [B][T][Hq])."""
    _need_cuda(o_parts, lse_parts, out, lse)
    if o_parts.dtype == torch.bfloat16:
        dt = TV_BF16
    elif o_parts.dtype == torch.float32:
        dt = TV_FP32
    else:
        raise TVError("o_parts must be bf16 or fp32")
    if not o_parts.is_contiguous() or not lse_parts.is_contiguous() or lse_parts.dtype != torch.float32:
        raise TVError("o_parts and lse_parts must be contiguous; lse_parts fp32")
    N, B, T, Hq, d = o_parts.shape
    if tuple(lse_parts.shape) != (N, B, T, Hq):
        raise TVError("lse_parts must be [N][B][T][Hq]")
    if out is None:
        out = torch.empty(B, T, Hq, d, dtype=o_parts.dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty(B, T, Hq, dtype=torch.float32, device=o_parts.device)
    if not out.is_contiguous() or out.dtype != o_parts.dtype or not lse.is_contiguous():
        raise TVError("out must be contiguous with o_parts' dtype; lse contiguous fp32")
    a = AttnMergeArgs(dt, N, B, T, Hq, d, o_parts.data_ptr(), lse_parts.data_ptr(), out.data_ptr(), lse.data_ptr())
    _check(lib().tree_verify_attn_merge(ctypes.byref(a), _stream(stream)), "tree_verify_attn_merge")
    return out, lse


# Which attention kernels the last tree_verify_attn call ran (tv_attn_path).
last_attn_path = None
last_attn_launches = None
ATTN_PATHS = {0: "cuda-core split-KV", 1: "tcgen05 prefix", 2: "block top-k sparse (cuda cores)",
              3: "block top-k sparse (tcgen05)", 4: "tcgen05 prefix, two query tiles per CTA",
              5: "tcgen05 prefix, two query tiles per CTA, chunks merged through the workspace"}


# --------------------------------------------------------------- KV commit

def tree_commit_kv(k_cache, v_cache, prefix_len, k_tree, v_tree, n_accepted, accepted_nodes,
                   dev_status=None, stream=None):
    """Append each sequence's accepted path (the root, then the accepted
    nodes) to its K/V cache and advance prefix_len in place
    (include/tree_verify.h, tree_commit_kv).  Shapes: caches [B][Lmax][Hkv][d],
    tree K/V [B][T][Hkv][d] (may be a view of the cache rows from
    prefix_len on), prefix_len and n_accepted [B] int32, accepted_nodes
    [B][T] int32 as tree_accept returns them."""
    dev = _need_cuda(k_cache, v_cache, prefix_len, k_tree, v_tree, n_accepted, accepted_nodes, dev_status)
    if k_cache.dtype == torch.bfloat16:
        dt = TV_BF16
    elif k_cache.dtype == torch.float32:
        dt = TV_FP32
    else:
        raise TVError("K/V must be bf16 or fp32")
    for t in (k_cache, v_cache, k_tree, v_tree):
        if t.dtype != k_cache.dtype or t.stride(-1) != 1:
            raise TVError("K/V must share one dtype with a contiguous last dimension")
    if k_cache.stride() != v_cache.stride() or k_tree.stride() != v_tree.stride():
        raise TVError("K and V tensors must have equal strides")
    B, Lmax, Hkv, d = k_cache.shape
    T = k_tree.shape[1]
    if tuple(k_tree.shape) != (B, T, Hkv, d) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise TVError("tree K/V must be [B][T][Hkv][d] and match the caches")
    prefix_len = _i32(prefix_len)
    n_accepted = _i32(n_accepted)
    if accepted_nodes.dtype != torch.int32 or accepted_nodes.stride(-1) != 1:
        raise TVError("accepted_nodes must be int32 with contiguous rows")
    a = CommitArgs(dt, B, T, Hkv, d, Lmax,
                   k_cache.data_ptr(), v_cache.data_ptr(), k_cache.stride(0), k_cache.stride(1), k_cache.stride(2),
                   prefix_len.data_ptr(),
                   k_tree.data_ptr(), v_tree.data_ptr(), k_tree.stride(0), k_tree.stride(1), k_tree.stride(2),
                   n_accepted.data_ptr(), accepted_nodes.data_ptr(), accepted_nodes.stride(0),
                   _ptr(dev_status))
    _check(lib().tree_commit_kv(ctypes.byref(a), _stream(stream)), "tree_commit_kv")
    return prefix_len


# --------------------------------------------------------------- acceptance

def tree_accept(target_logits, draft_tokens, parent, draft_probs=None, n_nodes=None,
                mode: str = "auto", temperature: float = 0.0, seed: int = 0, step: int = 0,
                dev_status=None, stream=None, outputs=None):
    """Acceptance walk (include/tree_verify.h, tree_accept).  target_logits
    and draft_probs are fp32 [B][T][V] with contiguous rows; draft_tokens and
    parent int32 [B][T].  Returns a dict of device tensors n_accepted [B],
    accepted_nodes [B][T], out_tokens [B][T+1], min_margin [B] (fp64)."""
    dev = _need_cuda(target_logits, draft_tokens, parent, draft_probs, n_nodes)
    B, T, V = target_logits.shape
    if target_logits.dtype != torch.float32 or target_logits.stride(-1) != 1:
        raise TVError("target_logits must be fp32 with contiguous rows")
    if draft_probs is not None and (draft_probs.dtype != torch.float32 or draft_probs.stride(-1) != 1):
        raise TVError("draft_probs must be fp32 with contiguous rows")
    for t in (draft_tokens, parent):
        if t.dtype != torch.int32 or t.stride(-1) != 1:
            raise TVError("draft_tokens / parent must be int32 with contiguous rows")
    n_nodes = _i32(n_nodes)
    if outputs is None:
        outputs = dict(n_accepted=torch.empty(B, dtype=torch.int32, device=dev),
                       accepted_nodes=torch.empty(B, T, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty(B, T + 1, dtype=torch.int32, device=dev),
                       min_margin=torch.empty(B, dtype=torch.float64, device=dev))
    o = outputs
    dp = draft_probs
    a = AcceptArgs(B, T, V,
                   target_logits.data_ptr(), target_logits.stride(0), target_logits.stride(1),
                   _ptr(dp), dp.stride(0) if dp is not None else 0, dp.stride(1) if dp is not None else 0,
                   draft_tokens.data_ptr(), draft_tokens.stride(0),
                   parent.data_ptr(), parent.stride(0),
                   _ptr(n_nodes), MODES[mode], float(temperature),
                   int(seed) & 0xFFFFFFFFFFFFFFFF, int(step) & 0xFFFFFFFFFFFFFFFF,
                   o["n_accepted"].data_ptr(), o["accepted_nodes"].data_ptr(), o["out_tokens"].data_ptr(),
                   _ptr(o.get("min_margin")), _ptr(dev_status))
    L = lib()
    need = L.tree_accept_workspace_size(ctypes.byref(a))
    sh = _stream(stream)
    ws = _workspace(dev, sh, need)
    _check(L.tree_accept(ctypes.byref(a), _aligned_ptr(ws), need, sh), "tree_accept")
    return o


def tree_accept_noalloc(target_logits, draft_tokens, parent, draft_probs=None, n_nodes=None,
                        mode: str = "auto", temperature: float = 0.0, seed: int = 0, step: int = 0,
                        dev_status=None, stream=None, outputs=None):
    """tree_accept without a workspace, for callers that cannot allocate
    device memory (include/tree_verify.h, tree_accept_noalloc): the library
    uses a fixed scratch array of its own (B * T <= 32768).  Only the
    outputs, when not given, are allocated here.  Calls that may overlap on
    the GPU share that scratch and must be serialised by the caller."""
    dev = _need_cuda(target_logits, draft_tokens, parent, draft_probs, n_nodes)
    B, T, V = target_logits.shape
    if target_logits.dtype != torch.float32 or target_logits.stride(-1) != 1:
        raise TVError("target_logits must be fp32 with contiguous rows")
    if draft_probs is not None and (draft_probs.dtype != torch.float32 or draft_probs.stride(-1) != 1):
        raise TVError("draft_probs must be fp32 with contiguous rows")
    for t in (draft_tokens, parent):
        if t.dtype != torch.int32 or t.stride(-1) != 1:
            raise TVError("draft_tokens / parent must be int32 with contiguous rows")
    n_nodes = _i32(n_nodes)
    if outputs is None:
        outputs = dict(n_accepted=torch.empty(B, dtype=torch.int32, device=dev),
                       accepted_nodes=torch.empty(B, T, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty(B, T + 1, dtype=torch.int32, device=dev),
                       min_margin=torch.empty(B, dtype=torch.float64, device=dev))
    o = outputs
    dp = draft_probs
    a = AcceptArgs(B, T, V,
                   target_logits.data_ptr(), target_logits.stride(0), target_logits.stride(1),
                   _ptr(dp), dp.stride(0) if dp is not None else 0, dp.stride(1) if dp is not None else 0,
                   draft_tokens.data_ptr(), draft_tokens.stride(0),
                   parent.data_ptr(), parent.stride(0),
                   _ptr(n_nodes), MODES[mode], float(temperature),
                   int(seed) & 0xFFFFFFFFFFFFFFFF, int(step) & 0xFFFFFFFFFFFFFFFF,
                   o["n_accepted"].data_ptr(), o["accepted_nodes"].data_ptr(), o["out_tokens"].data_ptr(),
                   _ptr(o.get("min_margin")), _ptr(dev_status))
    _check(lib().tree_accept_noalloc(ctypes.byref(a), _stream(stream)), "tree_accept_noalloc")
    return o


# --------------------------------------------------------------- expansion

class ExpandState:
    """Caller-owned device state of a best-first expansion (tree arrays and
    the candidate pool)."""

    def __init__(self, budget: int, V: int, Bsel: int, device):
        self.budget, self.V, self.Bsel = int(budget), int(V), int(Bsel)
        self.n_nodes = torch.zeros(1, dtype=torch.int32, device=device)
        self.parent = torch.full((budget,), -1, dtype=torch.int32, device=device)
        self.token = torch.full((budget,), -1, dtype=torch.int32, device=device)
        self.logp = torch.zeros(budget, dtype=torch.float64, device=device)
        nb = lib().tree_expand_pool_bytes(budget, V)
        self._pool = torch.zeros(nb + 256, dtype=torch.uint8, device=device)
        self.pool_bytes = nb
        self.frontier = torch.full((Bsel,), -1, dtype=torch.int32, device=device)
        self.n_appended = torch.zeros(1, dtype=torch.int32, device=device)

    @property
    def pool_ptr(self) -> int:
        return _aligned_ptr(self._pool)

    def args(self, draft_logits=None, row_node=None, temperature: float = 1.0, dev_status=None,
             mode: str = "bestfirst"):
        R = 0 if row_node is None else int(row_node.numel())
        ld = draft_logits.stride(0) if draft_logits is not None else self.V
        return ExpandArgs(self.V, R, self.Bsel, self.budget, float(temperature),
                          _ptr(draft_logits), ld, _ptr(row_node),
                          self.n_nodes.data_ptr(), self.parent.data_ptr(), self.token.data_ptr(),
                          self.logp.data_ptr(), self.pool_ptr, self.pool_bytes,
                          self.frontier.data_ptr(), self.n_appended.data_ptr(), _ptr(dev_status),
                          EXPAND_MODES[mode])


def tree_expand_init(budget: int, V: int, Bsel: int, root_token: int = 0, device=None,
                     state: Optional[ExpandState] = None, stream=None) -> ExpandState:
    """Allocate (or reset) an expansion state holding the root alone."""
    if state is None:
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        state = ExpandState(budget, V, Bsel, device)
    a = state.args()
    _check(lib().tree_expand_init(ctypes.byref(a), int(root_token), _stream(stream)), "tree_expand_init")
    return state


def tree_expand_topb(state: ExpandState, draft_logits, row_node, draft_temperature: float = 1.0,
                     dev_status=None, stream=None, mode: str = "bestfirst"):
    """One round (include/tree_verify.h, tree_expand_topb).  draft_logits fp32
    [R][V] with contiguous rows, row_node int32 [R]; mode "bestfirst"
    (batched best-first with a carried pool) or "beam" (the children of this
    round's rows only).  Returns the state's frontier and n_appended tensors
    (device)."""
    _need_cuda(draft_logits, row_node)
    if draft_logits.dtype != torch.float32 or draft_logits.stride(-1) != 1:
        raise TVError("draft_logits must be fp32 with contiguous rows")
    if mode not in EXPAND_MODES:
        raise TVError(f"mode must be one of {sorted(EXPAND_MODES)}")
    row_node = _i32(row_node)
    a = state.args(draft_logits, row_node, draft_temperature, dev_status, mode)
    _check(lib().tree_expand_topb(ctypes.byref(a), None, 0, _stream(stream)), "tree_expand_topb")
    return state.frontier, state.n_appended


# --------------------------------------------------------------- utilities

def philox_uniforms(seed: int, step: int, b, node, draw, tag, stream=None) -> torch.Tensor:
    """Device Philox uniforms of the acceptance walk for the given draws."""
    dev = _need_cuda(b, node, draw, tag)
    b, node, draw, tag = (_i32(x) for x in (b, node, draw, tag))
    out = torch.empty(b.numel(), dtype=torch.float64, device=dev)
    _check(lib().tv_philox_uniforms(int(seed) & 0xFFFFFFFFFFFFFFFF, int(step) & 0xFFFFFFFFFFFFFFFF,
                                    b.data_ptr(), node.data_ptr(), draw.data_ptr(), tag.data_ptr(),
                                    out.data_ptr(), b.numel(), _stream(stream)), "tv_philox_uniforms")
    return out


def expand_exp(t, stream=None) -> torch.Tensor:
    """The exponential of tree_expand_topb's fp64 log-sum-exp (tv_expand_exp):
    e^t for fp64 device t <= 0 (0 below -700)."""
    dev = _need_cuda(t)
    if t.dtype != torch.float64 or not t.is_contiguous():
        raise TVError("t must be contiguous fp64")
    out = torch.empty_like(t)
    _check(lib().tv_expand_exp(t.data_ptr(), out.data_ptr(), t.numel(), _stream(stream)), "tv_expand_exp")
    return out


def expand_set_wait_limit(polls: int) -> None:
    """Test hook (tv_expand_set_wait_limit): at most `polls` non-blocking
    tests per staged chunk in tree_expand_topb's row pass (0: default)."""
    _check(lib().tv_expand_set_wait_limit(int(polls)), "tv_expand_set_wait_limit")

