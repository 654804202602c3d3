"""Thin Python binding over libflide.so (include/flide.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  The
binding raises if the library is missing -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# FLIDE_DEBUG_BOUNDS=1 selects the bounds-checked build (build.py --debug-bounds)
LIB_PATH = os.path.join(_PKG, "libflide_dbg.so" if os.environ.get("FLIDE_DEBUG_BOUNDS") == "1"
                        else "libflide.so")

OK, ERR_INVALID, ERR_SHAPE, ERR_CAPACITY, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(7)
F32, BF16, E4M3 = 0, 1, 2
FLAG_PORTABLE = 1
COUNTS = 16
CNT = dict(N=0, T=1, PAST=2, DEPTH=3, SLOTS=4, BRANCH_TOK=5, ROOT_TOK=6, CKPT_ROWS=7,
           CHECK_SITE=12, CHECK_VALUE=13)

# names and order of the int32* members of flide_tree_index
INDEX_ARRAYS = ["status", "counts", "node_start", "node_req", "depth", "anc_ptr", "anc_node",
                "ctx_len", "token_node", "token_pos", "past_start", "req_node", "level_ptr",
                "level_node", "state_slot", "ckpt_start", "work"]

# every extern "C" symbol declared in include/flide.h
SYMBOLS = ["flide_tree_index_bytes", "flide_tree_index_init", "flide_tree_build",
           "flide_fork_attn", "flide_fork_attn_noalloc", "flide_fork_gdn", "flide_state_save",
           "flide_state_resume", "flide_branch_logprob_workspace_bytes", "flide_branch_logprob",
           "flide_option_probs", "flide_pool_create", "flide_pool_destroy", "flide_pool_append",
           "flide_pool_release", "flide_pool_length", "flide_pool_free_blocks", "flide_pool_export",
           "flide_history_append", "flide_history_gather", "flide_selftest_wait_timeout",
           "flide_fork_attn_fp8", "flide_amax", "flide_quantize_e4m3", "flide_fork_attn_paged",
           "flide_plan_state_groups", "flide_copy_rows", "flide_fork_gdn_fp8", "flide_pool_append_batch",
           "flide_tree_state_slots", "flide_debug_bounds", "flide_strerror"]


class FlideError(RuntimeError):
    def __init__(self, code, where=""):
        msg = _lib().flide_strerror(code).decode() if _LIB is not None else str(code)
        super().__init__(f"{where}: flide status {code} ({msg})")
        self.code = code


class TreeDesc(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int32), ("N", ctypes.c_int32), ("T", ctypes.c_int32),
                ("max_depth", ctypes.c_int32), ("req_node_ptr", ctypes.c_void_p),
                ("parent", ctypes.c_void_p), ("seg_len", ctypes.c_void_p),
                ("past_len", ctypes.c_void_p)]


class TreeIndexC(ctypes.Structure):
    _fields_ = ([("R", ctypes.c_int32), ("N", ctypes.c_int32), ("T", ctypes.c_int32),
                 ("max_depth", ctypes.c_int32)]
                + [(n, ctypes.c_void_p) for n in INDEX_ARRAYS]
                + [("work_len", ctypes.c_int64)])


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m tree_forked_decision_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        lib.flide_tree_index_bytes.argtypes = [I32, I32, I32, I32]
        lib.flide_tree_index_bytes.restype = ctypes.c_size_t
        lib.flide_tree_index_init.argtypes = [P, P, ctypes.c_size_t, I32, I32, I32, I32]
        lib.flide_tree_index_init.restype = ctypes.c_int
        lib.flide_tree_build.argtypes = [P, P, P]
        lib.flide_tree_build.restype = ctypes.c_int
        lib.flide_fork_attn.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32, F, P, I32, P]
        lib.flide_fork_attn.restype = ctypes.c_int
        lib.flide_fork_attn_noalloc.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32, F, P,
                                                I32, P]
        lib.flide_fork_attn_noalloc.restype = ctypes.c_int
        lib.flide_fork_gdn.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, P, P, I32, I32, P]
        lib.flide_fork_gdn.restype = ctypes.c_int
        lib.flide_state_save.argtypes = [P, P, P, P, P, I32, I32, I32, P, I32, I32, I32, P, P, P,
                                         I32, P]
        lib.flide_state_save.restype = ctypes.c_int
        lib.flide_state_resume.argtypes = [I32, P, I32, P, P, P, P, I32, I32, I32, I32, I32, I32,
                                           P, P, P, I32, P, P, P]
        lib.flide_state_resume.restype = ctypes.c_int
        lib.flide_branch_logprob_workspace_bytes.argtypes = [I32, I32]
        lib.flide_branch_logprob_workspace_bytes.restype = ctypes.c_size_t
        lib.flide_branch_logprob.argtypes = [P, P, P, P, I32, I32, I32, P, P, ctypes.c_size_t, P]
        lib.flide_branch_logprob.restype = ctypes.c_int
        lib.flide_option_probs.argtypes = [P, P, P, P, P]
        lib.flide_option_probs.restype = ctypes.c_int
        lib.flide_pool_create.argtypes = [I32, I32, I32, I32]
        lib.flide_pool_create.restype = P
        lib.flide_pool_destroy.argtypes = [P]
        lib.flide_pool_destroy.restype = None
        lib.flide_pool_append.argtypes = [P, I32, I32]
        lib.flide_pool_append.restype = ctypes.c_int64
        lib.flide_pool_append_batch.argtypes = [P, I32, P, P, P]
        lib.flide_pool_append_batch.restype = ctypes.c_int
        lib.flide_pool_release.argtypes = [P, I32]
        lib.flide_pool_release.restype = ctypes.c_int
        lib.flide_pool_length.argtypes = [P, I32]
        lib.flide_pool_length.restype = ctypes.c_int32
        lib.flide_pool_free_blocks.argtypes = [P]
        lib.flide_pool_free_blocks.restype = ctypes.c_int32
        lib.flide_pool_export.argtypes = [P, P, P]
        lib.flide_pool_export.restype = ctypes.c_int
        lib.flide_history_append.argtypes = [P, P, P, P, I32, I32, P, P, P, P, I32, I32, I32, P,
                                             I32, I32, I32, P, P]
        lib.flide_history_append.restype = ctypes.c_int
        lib.flide_history_gather.argtypes = [I32, P, I32, P, P, I32, I32, P, P, I32, I32, I32, P,
                                             I32, I32, I32, P, P, P, I32, P, P, P]
        lib.flide_history_gather.restype = ctypes.c_int
        lib.flide_selftest_wait_timeout.argtypes = [P, I32, I32, P]
        lib.flide_selftest_wait_timeout.restype = ctypes.c_int
        lib.flide_fork_attn_fp8.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, P, F, P, P]
        lib.flide_fork_attn_fp8.restype = ctypes.c_int
        lib.flide_fork_attn_paged.argtypes = [P, P, P, P, P, I32, I32, P, I32, P, I32, P, I32, I32,
                                              I32, I32, P, F, P, P]
        lib.flide_fork_attn_paged.restype = ctypes.c_int
        lib.flide_plan_state_groups.argtypes = [I32, P, P, I32, P, P]
        lib.flide_plan_state_groups.restype = ctypes.c_int
        lib.flide_tree_state_slots.argtypes = [I32, P, P, P]
        lib.flide_tree_state_slots.restype = ctypes.c_int
        lib.flide_copy_rows.argtypes = [P, P, P, P, I32, ctypes.c_int64, P]
        lib.flide_copy_rows.restype = ctypes.c_int
        lib.flide_fork_gdn_fp8.argtypes = [P, P, P, P, P, P, P, P, I32, I32, I32, P, P, I32, P]
        lib.flide_fork_gdn_fp8.restype = ctypes.c_int
        lib.flide_amax.argtypes = [P, ctypes.c_int64, I32, P, I32, P]
        lib.flide_amax.restype = ctypes.c_int
        lib.flide_quantize_e4m3.argtypes = [P, ctypes.c_int64, I32, P, P, P, P]
        lib.flide_quantize_e4m3.restype = ctypes.c_int
        lib.flide_debug_bounds.argtypes = []
        lib.flide_debug_bounds.restype = ctypes.c_int32
        lib.flide_strerror.argtypes = [ctypes.c_int32]
        lib.flide_strerror.restype = ctypes.c_char_p
        _LIB = lib
    return _LIB


def load():
    """Loads libflide.so (raises if absent) and returns the ctypes handle."""
    return _lib()


def _check(code, where):
    if code != OK:
        raise FlideError(code, where)


def _ptr(t):
    """Device address of a tensor for the C ABI.  The kernels index dense
    row-major device arrays, so a strided view or a host tensor is refused
    here (a host address handed to a kernel would fault the GPU)."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got strides {tuple(t.stride())} "
                         f"for shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


class TreeIndex:
    """Device-resident tree index over one torch-allocated buffer."""

    def __init__(self, R: int, N: int, T: int, max_depth: int, device="cuda"):
        lib = _lib()
        nbytes = lib.flide_tree_index_bytes(R, N, T, max_depth)
        if nbytes == 0:
            raise FlideError(ERR_SHAPE, "flide_tree_index_bytes")
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.c = TreeIndexC()
        _check(lib.flide_tree_index_init(ctypes.byref(self.c), ctypes.c_void_p(self.buf.data_ptr()),
                                         nbytes, R, N, T, max_depth), "flide_tree_index_init")
        self.R, self.N, self.T, self.max_depth = R, N, T, max_depth

    def array(self, name: str, n: int) -> torch.Tensor:
        """int32 view of one index array (first n entries)."""
        off = getattr(self.c, name) - self.buf.data_ptr()
        return self.buf[off:off + 4 * n].view(torch.int32)

    def status(self) -> int:
        return int(self.array("status", 1).item())

    def counts(self) -> dict:
        c = self.array("counts", COUNTS).cpu().tolist()
        return {k: c[v] for k, v in CNT.items()}


class DeviceTree:
    """Device copies of a tree's arrays (the flide_tree_desc inputs)."""

    def __init__(self, req_node_ptr, parent, seg_len, past_len, max_depth: int,
                 N: int | None = None, T: int | None = None, device="cuda"):
        as_i32 = lambda a: torch.as_tensor(np.asarray(a, np.int32)).to(device)
        self._host = tuple(np.asarray(a, np.int32) for a in (req_node_ptr, parent, seg_len, past_len))
        self.req_node_ptr = as_i32(req_node_ptr)
        self.parent = as_i32(parent)
        self.seg_len = as_i32(seg_len)
        self.past_len = as_i32(past_len)
        self.R = len(req_node_ptr) - 1
        self.N = int(N if N is not None else max(len(parent), 1))
        self.T = int(T if T is not None else max(int(np.sum(seg_len)), 1))
        self.max_depth = int(max_depth)
        if len(parent) == 0:  # keep valid pointers for empty batches
            self.parent = torch.full((1,), -1, dtype=torch.int32, device=device)
            self.seg_len = torch.zeros(1, dtype=torch.int32, device=device)

    @classmethod
    def from_buffers(cls, req_node_ptr, parent, seg_len, past_len, N: int, T: int,
                     max_depth: int) -> "DeviceTree":
        """Wraps preallocated int32 device buffers (capacities N, T) without copying."""
        t = cls.__new__(cls)
        t._host = None
        t.req_node_ptr, t.parent, t.seg_len, t.past_len = req_node_ptr, parent, seg_len, past_len
        t.R = req_node_ptr.shape[0] - 1
        t.N, t.T, t.max_depth = int(N), int(T), int(max_depth)
        return t

    def arrays(self):
        """The host arrays (req_node_ptr, parent, seg_len, past_len) the tree was
        built from (for host-side sizing such as state_slots)."""
        if self._host is None:
            raise ValueError("a DeviceTree wrapping device buffers has no host arrays")
        return self._host

    def desc(self) -> TreeDesc:
        return TreeDesc(self.R, self.N, self.T, self.max_depth, self.req_node_ptr.data_ptr(),
                        self.parent.data_ptr(), self.seg_len.data_ptr(), self.past_len.data_ptr())


def tree_build(tree: DeviceTree, index: TreeIndex, stream=None):
    d = tree.desc()
    _check(_lib().flide_tree_build(ctypes.byref(d), ctypes.byref(index.c), _stream(stream)),
           "flide_tree_build")



def _attn_args(where, q, k, v, past_k, past_v, out):
    """q [T, Hq, d]; k, v [T, Hkv, d]; past_k, past_v [P, Hkv, d]; out like q;
    one element type for all (the library reads every tensor as q's type)."""
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or k.shape[0] != q.shape[0] \
            or k.shape[2] != q.shape[2]:
        raise ValueError(f"{where}: expected q [T, Hq, d] and k, v [T, Hkv, d], got "
                         f"{tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    for name, t in (("k", k), ("v", v), ("past_k", past_k), ("past_v", past_v), ("out", out)):
        if t is not None and t.dtype != q.dtype:
            raise TypeError(f"{where}: {name} is {t.dtype}, q is {q.dtype}")
    if past_k is not None and past_v is not None and (
            past_k.shape != past_v.shape or past_k.dim() != 3 or past_k.shape[1:] != k.shape[1:]):
        raise ValueError(f"{where}: expected past_k, past_v [P, Hkv, d]")
    if out.shape != q.shape:
        raise ValueError(f"{where}: out must have q's shape {tuple(q.shape)}")


def _bf16_out(where, out, shape):
    if out.dtype != torch.bfloat16 or tuple(out.shape) != tuple(shape):
        raise TypeError(f"{where}: out must be bfloat16 {tuple(shape)}")


def _gdn_args(where, q, k, v, g, beta, state_in, node_state, out):
    """q, k [T, H, dk]; v, out [T, H, dv] of q's element type; g, beta [T, H]
    float32; state_in [R, H, dv, dk] and node_state [slots, H, dv, dk] float32."""
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError(f"{where}: expected q, k [T, H, dk] and v [T, H, dv], got "
                         f"{tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    for name, t in (("k", k), ("v", v), ("out", out)):
        if t.dtype != q.dtype:
            raise TypeError(f"{where}: {name} is {t.dtype}, q is {q.dtype}")
    for name, t in (("g", g), ("beta", beta)):
        if t.dtype != torch.float32 or t.shape != q.shape[:2]:
            raise TypeError(f"{where}: {name} must be float32 [T, H]")
    T, H, dk = q.shape
    dv = v.shape[2]
    for name, t in (("state_in", state_in), ("node_state", node_state)):
        if t is not None and (t.dtype != torch.float32 or t.dim() != 4 or tuple(t.shape[1:]) != (H, dv, dk)):
            raise TypeError(f"{where}: {name} must be float32 [*, {H}, {dv}, {dk}]")
    if tuple(out.shape) != (T, H, dv):
        raise ValueError(f"{where}: out must be [{T}, {H}, {dv}]")


def fork_attn(q, k, v, index: TreeIndex, scale: float, past_k=None, past_v=None, out=None,
              flags: int = 0, stream=None):
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    past_rows = 0 if past_k is None else past_k.shape[0]
    if past_rows == 0:
        past_k = past_v = None
    _attn_args("fork_attn", q, k, v, past_k, past_v, out)
    _check(_lib().flide_fork_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(past_k), _ptr(past_v),
                                  past_rows, ctypes.byref(index.c), Hq, Hkv, d, _dtype_code(q),
                                  float(scale), _ptr(out), flags, _stream(stream)),
           "flide_fork_attn")
    return out


def fork_attn_fp8(q8, k8, v8, index: TreeIndex, scale: float, descale, past_k=None, past_v=None,
                  out=None, stream=None):
    """Fork attention over e4m3 codes (uint8 tensors [T, H, 128]); descale is
    a float32 device tensor [3] = (sq, sk, sv); past rows use sk and sv.
    Returns bf16 [T, Hq, 128]."""
    T, Hq, d = q8.shape
    Hkv = k8.shape[1]
    for t in (q8, k8, v8, past_k, past_v):
        if t is not None and (t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous()):
            raise TypeError("e4m3 inputs must be contiguous uint8 / float8_e4m3fn tensors")
    if descale.dtype != torch.float32 or descale.numel() < 3:
        raise TypeError("descale must be a float32 tensor of 3 entries")
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=q8.device)
    _bf16_out("fork_attn_fp8", out, (T, Hq, d))
    past_rows = 0 if past_k is None else past_k.shape[0]
    if past_rows == 0:
        past_k = past_v = None
    _check(_lib().flide_fork_attn_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(past_k), _ptr(past_v),
                                      past_rows, ctypes.byref(index.c), Hq, Hkv, d, _ptr(descale),
                                      float(scale), _ptr(out), _stream(stream)),
           "flide_fork_attn_fp8")
    return out


def fork_attn_paged(q, k, v, index: TreeIndex, scale: float, pool_k, pool_v, block_table,
                    req_slot, block_rows: int, max_blocks: int, descale=None, out=None,
                    stream=None):
    """Fork attention with each request's past rows read in place from a
    block-paged pool (pool_k/pool_v [n_blocks * block_rows, Hkv, 128], bf16 or
    e4m3 codes with descale), block_table int32 [n_slots * max_blocks],
    req_slot int32 [R] on the device.  Returns bf16 [T, Hq, 128]."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    e4m3 = q.dtype in (torch.uint8, torch.float8_e4m3fn)
    dtype = E4M3 if e4m3 else _dtype_code(q)
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=q.device)
    _bf16_out("fork_attn_paged", out, (T, Hq, d))
    byte = lambda t: torch.uint8 if t.dtype == torch.float8_e4m3fn else t.dtype  # e4m3 codes
    for name, t in (("k", k), ("v", v), ("pool_k", pool_k), ("pool_v", pool_v)):
        if byte(t) != byte(q):
            raise TypeError(f"fork_attn_paged: {name} is {t.dtype}, q is {q.dtype}")
    if pool_v.shape != pool_k.shape or pool_k.dim() != 3 or pool_k.shape[1:] != k.shape[1:]:
        raise ValueError("fork_attn_paged: pools must be [n_blocks * block_rows, Hkv, d]")
    for name, t in (("block_table", block_table), ("req_slot", req_slot)):
        if t.dtype != torch.int32:
            raise TypeError(f"fork_attn_paged: {name} must be int32")
    n_blocks = pool_k.shape[0] // block_rows
    n_slots = block_table.numel() // max_blocks
    _check(_lib().flide_fork_attn_paged(_ptr(q), _ptr(k), _ptr(v), _ptr(pool_k), _ptr(pool_v),
                                        n_blocks, block_rows, _ptr(block_table), max_blocks,
                                        _ptr(req_slot), n_slots, ctypes.byref(index.c), Hq, Hkv, d,
                                        dtype, _ptr(descale), float(scale), _ptr(out),
                                        _stream(stream)),
           "flide_fork_attn_paged")
    return out


def fork_gdn_fp8(q8, k8, v8, g, beta, index: TreeIndex, node_state, descale, state_in=None,
                 out=None, stream=None):
    """GDN fork scan over e4m3 codes (uint8 tensors q, k [T, H, 128], v
    [T, H, 128]); descale is a float32 device tensor [3] = (sq, sk, sv).
    Returns bf16 [T, H, 128]."""
    T, H, dk = q8.shape
    dv = v8.shape[2]
    for t in (q8, k8, v8):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous():
            raise TypeError("e4m3 inputs must be contiguous uint8 / float8_e4m3fn tensors")
    if descale.dtype != torch.float32 or descale.numel() < 3:
        raise TypeError("descale must be a float32 tensor of 3 entries")
    if out is None:
        out = torch.empty((T, H, dv), dtype=torch.bfloat16, device=q8.device)
    _bf16_out("fork_gdn_fp8", out, (T, H, dv))
    for name, t in (("g", g), ("beta", beta)):
        if t.dtype != torch.float32 or t.shape != q8.shape[:2]:
            raise TypeError(f"fork_gdn_fp8: {name} must be float32 [T, H]")
    for name, t in (("state_in", state_in), ("node_state", node_state)):
        if t is not None and (t.dtype != torch.float32 or t.dim() != 4 or tuple(t.shape[1:]) != (H, dv, dk)):
            raise TypeError(f"fork_gdn_fp8: {name} must be float32 [*, {H}, {dv}, {dk}]")
    _check(_lib().flide_fork_gdn_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(descale), _ptr(g),
                                     _ptr(beta), _ptr(state_in), ctypes.byref(index.c), H, dk, dv,
                                     _ptr(out), _ptr(node_state), node_state.shape[0],
                                     _stream(stream)), "flide_fork_gdn_fp8")
    return out


def amax(x, out=None, accumulate: bool = False, stream=None):
    """float32 device tensor [1] = max |x| (max with its current value when
    accumulate), for per-tensor e4m3 scaling."""
    if not x.is_contiguous():
        raise TypeError("x must be contiguous")
    if out is None:
        out = torch.zeros(1, dtype=torch.float32, device=x.device)
    _check(_lib().flide_amax(_ptr(x), x.numel(), _dtype_code(x), _ptr(out), int(bool(accumulate)),
                             _stream(stream)), "flide_amax")
    return out


def quantize_e4m3(x, amax_t=None, out=None, descale=None, stream=None):
    """e4m3 codes of x (uint8, x's shape) scaled so that amax_t (default: x's
    own absolute maximum) maps to 448, and the descale factor amax / 448
    (float32 device tensor [1])."""
    if not x.is_contiguous():
        raise TypeError("x must be contiguous")
    if amax_t is None:
        amax_t = amax(x, stream=stream)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if descale is None:
        descale = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(_lib().flide_quantize_e4m3(_ptr(x), x.numel(), _dtype_code(x), _ptr(amax_t), _ptr(out),
                                      _ptr(descale), _stream(stream)), "flide_quantize_e4m3")
    return out, descale


def fork_attn_noalloc(q, k, v, index: TreeIndex, scale: float, past_k=None, past_v=None,
                      out=None, flags: int = 0, stream=None):
    """flide_fork_attn_noalloc: same result as fork_attn, for callers that cannot
    provide scratch; leaves index.c.work untouched and allocates nothing."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    past_rows = 0 if past_k is None else past_k.shape[0]
    if past_rows == 0:
        past_k = past_v = None
    _attn_args("fork_attn_noalloc", q, k, v, past_k, past_v, out)
    _check(_lib().flide_fork_attn_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(past_k), _ptr(past_v),
                                          past_rows, ctypes.byref(index.c), Hq, Hkv, d,
                                          _dtype_code(q), float(scale), _ptr(out), flags,
                                          _stream(stream)),
           "flide_fork_attn_noalloc")
    return out


def fork_gdn(q, k, v, g, beta, index: TreeIndex, node_state, state_in=None, out=None,
             flags: int = 0, stream=None):
    T, H, dk = q.shape
    dv = v.shape[2]
    if out is None:
        out = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    _gdn_args("fork_gdn", q, k, v, g, beta, state_in, node_state, out)
    _check(_lib().flide_fork_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
                                 ctypes.byref(index.c), H, dk, dv, _dtype_code(q), _ptr(out),
                                 _ptr(node_state), node_state.shape[0], flags, _stream(stream)),
           "flide_fork_gdn")
    return out


def _rows_like(where, ref, **named):
    """K/V row tensors copied with ref's element type and row layout."""
    for name, t in named.items():
        if t is not None and (t.dtype != ref.dtype or t.dim() != 3 or t.shape[1:] != ref.shape[1:]):
            raise TypeError(f"{where}: {name} must be {ref.dtype} [*, {ref.shape[1]}, {ref.shape[2]}]")


def _states_like(where, H, dv, dk, **named):
    for name, t in named.items():
        if t is not None and (t.dtype != torch.float32 or t.dim() != 4
                              or tuple(t.shape[1:]) != (H, dv, dk)):
            raise TypeError(f"{where}: {name} must be float32 [*, {H}, {dv}, {dk}]")


def _int32(where, **named):
    for name, t in named.items():
        if t is not None and t.dtype != torch.int32:
            raise TypeError(f"{where}: {name} must be int32")


def state_save(index: TreeIndex, k, v, ckpt_k, ckpt_v, ckpt_S, past_k=None, past_v=None,
               node_state=None, stream=None):
    Hkv, d = (k.shape[1], k.shape[2]) if k is not None else (0, 0)
    H = dv = dk = 0
    if node_state is not None:
        _, H, dv, dk = node_state.shape
    dt = _dtype_code(k) if k is not None else BF16
    if k is not None:
        _rows_like("state_save", k, v=v, ckpt_k=ckpt_k, ckpt_v=ckpt_v, past_k=past_k, past_v=past_v)
    if node_state is not None:
        _states_like("state_save", H, dv, dk, node_state=node_state, ckpt_S=ckpt_S)
    _check(_lib().flide_state_save(ctypes.byref(index.c), _ptr(k), _ptr(v), _ptr(past_k),
                                   _ptr(past_v), Hkv, d, dt, _ptr(node_state), H, dk, dv,
                                   _ptr(ckpt_k), _ptr(ckpt_v), _ptr(ckpt_S),
                                   0 if ckpt_k is None else ckpt_k.shape[0], _stream(stream)),
           "flide_state_save")


def state_resume(src_req, src_ckpt_start, src_k, src_v, src_S, past_len, past_k, past_v,
                 state_in, status, stream=None):
    R = src_req.shape[0]
    src_R = src_ckpt_start.shape[0] - 1
    Hkv, d = src_k.shape[1], src_k.shape[2]
    H = dv = dk = 0
    if state_in is not None:
        _, H, dv, dk = state_in.shape
        _states_like("state_resume", H, dv, dk, src_S=src_S, state_in=state_in)
    _rows_like("state_resume", src_k, src_v=src_v, past_k=past_k, past_v=past_v)
    _int32("state_resume", src_req=src_req, src_ckpt_start=src_ckpt_start, past_len=past_len,
           status=status)
    _check(_lib().flide_state_resume(R, _ptr(src_req), src_R, _ptr(src_ckpt_start), _ptr(src_k),
                                     _ptr(src_v), _ptr(src_S), Hkv, d, _dtype_code(src_k), H, dk,
                                     dv, _ptr(past_len), _ptr(past_k), _ptr(past_v),
                                     past_k.shape[0], _ptr(state_in), _ptr(status),
                                     _stream(stream)),
           "flide_state_resume")


def selftest_wait_timeout(status, timeout_us: int, arrive: bool = False, stream=None):
    """The library's bounded device wait on a barrier nothing arrives at
    (diagnostic): FLIDE_ERR_TIMEOUT lands in `status` after `timeout_us`; with
    arrive=True the wait completes at once and `status` is left alone."""
    _check(_lib().flide_selftest_wait_timeout(_ptr(status), int(timeout_us), 1 if arrive else 0,
                                              _stream(stream)),
           "flide_selftest_wait_timeout")


def branch_logprob_workspace(index: TreeIndex, V: int, device="cuda") -> torch.Tensor:
    n = int(_lib().flide_branch_logprob_workspace_bytes(index.T, int(V)))
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def branch_logprob(h, w_lm, targets, index: TreeIndex, logp=None, workspace=None, stream=None):
    """log p(target) of every branch token under the LM head w_lm [V, D];
    h [T, D] (or [T, heads, dim]) bf16, targets [T] int32.  Root tokens: NaN."""
    T = h.shape[0]
    D = h[0].numel()
    V = w_lm.shape[0]
    if logp is None:
        logp = torch.empty(T, dtype=torch.float32, device=h.device)
    if workspace is None:
        workspace = branch_logprob_workspace(index, V, device=h.device)
    if w_lm.dtype != h.dtype or w_lm.dim() != 2 or w_lm.shape[1] != D:
        raise TypeError(f"branch_logprob: w_lm must be {h.dtype} [V, {D}]")
    _int32("branch_logprob", targets=targets)
    if targets.numel() < T or logp.dtype != torch.float32 or logp.numel() < T:
        raise ValueError(f"branch_logprob: targets (int32) and logp (float32) need {T} entries")
    _check(_lib().flide_branch_logprob(_ptr(h), _ptr(w_lm), _ptr(targets), ctypes.byref(index.c), D, V,
                                       _dtype_code(h), _ptr(logp), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)),
           "flide_branch_logprob")
    return logp


def option_probs(index: TreeIndex, logp, path_logp=None, prob=None, stream=None):
    """Per node: path log-likelihood and, for leaves, the softmax over the
    request's leaves (the decision distribution)."""
    N = index.N
    if path_logp is None:
        path_logp = torch.empty(max(N, 1), dtype=torch.float32, device=logp.device)
    if prob is None:
        prob = torch.empty(max(N, 1), dtype=torch.float32, device=logp.device)
    for name, t in (("logp", logp), ("path_logp", path_logp), ("prob", prob)):
        if t.dtype != torch.float32:
            raise TypeError(f"option_probs: {name} must be float32")
    if path_logp.numel() < N or prob.numel() < N:
        raise ValueError(f"option_probs: path_logp and prob need {N} entries")
    _check(_lib().flide_option_probs(ctypes.byref(index.c), _ptr(logp), _ptr(path_logp), _ptr(prob),
                                     _stream(stream)),
           "flide_option_probs")
    return path_logp, prob


def state_slots(tree) -> int:
    """Node-state slots that flide_tree_build assigns to a tree (counts["SLOTS"]),
    from the library's host query flide_tree_state_slots."""
    rp, parent, _seg, _past = tree.arrays()
    rp32 = np.ascontiguousarray(rp, np.int32)
    pa32 = np.ascontiguousarray(parent, np.int32)
    slots = ctypes.c_int32(0)
    _check(_lib().flide_tree_state_slots(len(rp32) - 1, rp32.ctypes.data_as(ctypes.c_void_p),
                                         pa32.ctypes.data_as(ctypes.c_void_p), ctypes.byref(slots)),
           "flide_tree_state_slots")
    return int(slots.value)
