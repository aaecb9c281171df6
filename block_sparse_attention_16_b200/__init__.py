"""Python binding of liblbsa (block-sparse self-attention over 3D video token grids, sm_100a).

Argument marshalling only: every step runs in the library's CUDA kernels;
torch supplies device memory and the current stream.  The functions carry the
C ABI's names (``include/lbsa.h``):

    scores          = lbsa_score(q, k, block, mode="exact")      # [B,H,nB,nB] fp32
    bs              = lbsa_select(scores, block, p=0.99, scope="row")
    out             = lbsa_attend(q, k, v, bs)                  # same shape/dtype as q
    row_ptr, col    = lbsa_blockset_export(bs)
    bits            = lbsa_blockset_export_bitmask(bs)          # [B,H,nB,ceil(nB/32)] block bits
    scores, out     = lbsa_score_attend(q, k, v, block)          # dense step: O and exact masses
    perm            = lbsa_partition_perm(T, H, W, "3d", tile=(4, 4, 4))
    qp, kp, vp      = lbsa_permute([q, k, v], perm)

Tensors are [B, H, N_valid, d] with a contiguous last dim, bf16 or fp32, on
the current CUDA device.  There is no CPU fallback: a missing library or a
missing GPU raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "LbsaError", "Blockset", "lbsa_score", "lbsa_select", "lbsa_attend", "lbsa_free",
    "lbsa_blockset_info", "lbsa_blockset_export", "lbsa_blockset_from_csr", "lbsa_get_status",
    "lbsa_device_status", "lbsa_partition_perm", "lbsa_permute", "lbsa_selftest_wait", "lbsa_selftest_exp2", "lbsa_select_rule", "lbsa_score_attend",
    "lbsa_select_head_noalloc", "lbsa_select_tokens", "lbsa_select_routed", "lbsa_blockset_views",
    "lbsa_blockset_masks", "lbsa_blockset_export_bitmask", "lbsa_blockset_from_bitmask",
    "lbsa_last_error", "lbsa_version", "library_path", "load_library",
    "LBSA_OK", "LBSA_ERR_INVALID_ARG", "LBSA_ERR_UNSUPPORTED", "LBSA_ERR_CUDA", "LBSA_ERR_OOM",
    "LBSA_ERR_BAD_INDEX", "LBSA_ERR_INVALID_SCORES", "LBSA_ERR_TIMEOUT",
]

LBSA_OK, LBSA_ERR_INVALID_ARG, LBSA_ERR_UNSUPPORTED, LBSA_ERR_CUDA = 0, 1, 2, 3
LBSA_ERR_OOM, LBSA_ERR_BAD_INDEX, LBSA_ERR_INVALID_SCORES, LBSA_ERR_TIMEOUT = 4, 5, 6, 7
_MODES = {"exact": 0, "meanpool": 1, "meanpool_token": 2}
_SCOPES = {"row": 0, "head": 1}
_PARTS = {"raster": 0, "1d": 1, "2d": 2, "3d": 3}


class LbsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"lbsa error {code}: {msg}")
        self.code = code


class _Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N_valid", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64), ("stride_n", ctypes.c_int64)]


_LIB = None


def library_path() -> str:
    """The in-tree liblbsa.so, or the file named by the LBSA_LIBRARY environment variable."""
    return os.environ.get("LBSA_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblbsa.so")


def load_library():
    """Load liblbsa.so (built by ``build.py``); raises if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise LbsaError(LBSA_ERR_UNSUPPORTED,
                        f"{path} not built: run python -m block_sparse_attention_16_b200.build")
    lib = ctypes.CDLL(path)
    P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    sig = {
        "lbsa_score": (ctypes.c_int, [P, P, ctypes.POINTER(_Desc), I32, I32, P, P, P]),
        "lbsa_select": (ctypes.c_int, [P, I32, I32, I32, I32, D, I32, ctypes.POINTER(P), P]),
        "lbsa_select_rule": (ctypes.c_int, [P, I32, I32, I32, I32, I32, I32, D, I32, ctypes.POINTER(P), P]),
        "lbsa_score_attend": (ctypes.c_int, [P, P, P, ctypes.POINTER(_Desc), I32, P, P, P, P]),
        "lbsa_attend": (ctypes.c_int, [P, P, P, ctypes.POINTER(_Desc), P, P, P, P]),
        "lbsa_free": (None, [P]),
        "lbsa_blockset_info": (ctypes.c_int, [P] + [ctypes.POINTER(I32)] * 5),
        "lbsa_blockset_views": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P)]),
        "lbsa_blockset_masks": (ctypes.c_int, [P, ctypes.POINTER(P)]),
        "lbsa_select_tokens": (ctypes.c_int, [P, I32, I32, I32, I32, D, ctypes.POINTER(P), P]),
        "lbsa_select_routed": (ctypes.c_int, [P, I32, I32, I32, I32, D, D, I32, P, P, ctypes.POINTER(P), P]),
        "lbsa_blockset_export": (ctypes.c_int, [P, P, P, ctypes.POINTER(I64), P]),
        "lbsa_blockset_from_csr": (ctypes.c_int, [P, P, I32, I32, I32, I32, ctypes.POINTER(P), P]),
        "lbsa_blockset_export_bitmask": (ctypes.c_int, [P, P, P]),
        "lbsa_blockset_from_bitmask": (ctypes.c_int, [P, I32, I32, I32, I32, ctypes.POINTER(P), P]),
        "lbsa_get_status": (ctypes.c_int, [P, ctypes.POINTER(I32), I32, P]),
        "lbsa_device_status": (ctypes.c_int, [ctypes.POINTER(I32), I32, P]),
        "lbsa_partition_perm": (ctypes.c_int, [I32, I32, I32, I32, I32, I32, I32, P, I32, P]),
        "lbsa_permute": (ctypes.c_int, [ctypes.POINTER(P), ctypes.POINTER(P), I32, P,
                                        ctypes.POINTER(_Desc), I32, P]),
        "lbsa_selftest_wait": (ctypes.c_int, [I64, P, P]),
        "lbsa_selftest_exp2": (ctypes.c_int, [P, P, I64, P]),
        "lbsa_select_head_noalloc": (ctypes.c_int, [P, I32, I32, I32, D, P, P, P, P]),
        "lbsa_last_error": (ctypes.c_char_p, []),
        "lbsa_version": (ctypes.c_int, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def _check(rc: int):
    if rc != LBSA_OK:
        raise LbsaError(rc, load_library().lbsa_last_error().decode())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _desc(x: torch.Tensor) -> _Desc:
    if x.dim() != 4 or x.stride(-1) != 1:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "expected [B, H, N, d] with a contiguous last dim")
    _on_device(x, "q", contiguous=False)
    if x.dtype == torch.bfloat16:
        dt = 0
    elif x.dtype == torch.float32:
        dt = 1
    else:
        raise LbsaError(LBSA_ERR_UNSUPPORTED, f"dtype {x.dtype}")
    B, H, N, d = x.shape
    return _Desc(B, H, N, d, dt, 0, x.stride(0), x.stride(1), x.stride(2))


def _on_device(x, name: str, dtype=None, min_numel: int = 0, contiguous: bool = True):
    """The library reads and writes only device memory of the current CUDA
    device: reject anything else before a pointer reaches it."""
    if x is None:
        return
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if x.device.index != torch.cuda.current_device():
        raise LbsaError(LBSA_ERR_INVALID_ARG,
                        f"{name} lives on cuda:{x.device.index}, the current device is cuda:{torch.cuda.current_device()}")
    if dtype is not None and x.dtype != dtype:
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"{name} must be {dtype}, got {x.dtype}")
    if contiguous and not x.is_contiguous():
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if x.numel() < min_numel:
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"{name} holds {x.numel()} elements, {min_numel} needed")


def _same_layout(a: torch.Tensor, b: torch.Tensor):
    if a.shape != b.shape or a.stride() != b.stride() or a.dtype != b.dtype or a.device != b.device:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "q, k, v (and out) must share shape, strides, dtype and device")


class Blockset:
    """Owner of a library blockset handle (freed with lbsa_free)."""

    def __init__(self, handle: int, keep=()):
        self.handle = ctypes.c_void_p(handle)
        self._keep = keep
        B, H, nB, blk, sc = (ctypes.c_int32() for _ in range(5))
        _check(load_library().lbsa_blockset_info(self.handle, ctypes.byref(B), ctypes.byref(H),
                                                 ctypes.byref(nB), ctypes.byref(blk), ctypes.byref(sc)))
        self.B, self.H, self.nB, self.block, self.scope = B.value, H.value, nB.value, blk.value, sc.value

    def free(self):
        if self.handle:
            load_library().lbsa_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def lbsa_score(q, k, block: int, mode: str = "exact", scores=None, lse=None, want_lse=False, stream=None):
    """Block scores [B, H, nB, nB] fp32 (and the dense row lse when asked, exact mode);
    mode "meanpool_token" scores every query token: [B, H, N, nB]."""
    _same_layout(q, k)
    desc = _desc(q)
    B, H, N, _ = q.shape
    nB = -(-N // block)
    if scores is None:
        scores = torch.empty(B, H, N if mode == "meanpool_token" else nB, nB, dtype=torch.float32, device=q.device)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _on_device(scores, "scores", torch.float32, B * H * (N if mode == "meanpool_token" else nB) * nB)
    _on_device(lse, "lse", torch.float32, B * H * N)
    _check(load_library().lbsa_score(_ptr(q), _ptr(k), ctypes.byref(desc), block, _MODES[mode],
                                     _ptr(scores), _ptr(lse), _stream(stream)))
    return (scores, lse) if (want_lse or lse is not None) else scores


def lbsa_select(scores, block: int, p: float = 0.99, scope: str = "row", stream=None) -> Blockset:
    """Mass-threshold selection of fp32 scores [B, H, nB, nB] into a new blockset."""
    _on_device(scores, "scores")
    if scores.dtype != torch.float32 or not scores.is_contiguous() or scores.dim() != 4:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be a contiguous fp32 [B, H, nB, nB] tensor")
    B, H, nB, nB2 = scores.shape
    if nB != nB2:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be square per head")
    h = ctypes.c_void_p()
    _check(load_library().lbsa_select(_ptr(scores), B, H, nB, block, float(p), _SCOPES[scope],
                                      ctypes.byref(h), _stream(stream)))
    return Blockset(h.value)


def lbsa_select_tokens(scores, block: int = 64, p: float = 0.25, stream=None) -> Blockset:
    """Head-scope selection over the (query token, key block) pairs of fp32
    scores [B, H, N, nB] into a new per-token blockset (64-token blocks)."""
    _on_device(scores, "scores")
    if scores.dtype != torch.float32 or not scores.is_contiguous() or scores.dim() != 4:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be a contiguous fp32 [B, H, N, nB] tensor")
    B, H, N, nB = scores.shape
    if nB != -(-N // block):
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"scores have {nB} key blocks, {N} tokens need {-(-N // block)}")
    h = ctypes.c_void_p()
    _check(load_library().lbsa_select_tokens(_ptr(scores), B, H, N, block, float(p), ctypes.byref(h),
                                             _stream(stream)))
    return Blockset(h.value)


class _DeviceArray:
    """A device buffer of the library seen through __cuda_array_interface__."""

    def __init__(self, ptr: int, n: int, typestr: str):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr, "data": (ptr, False), "version": 3}


def lbsa_blockset_views(bs: Blockset):
    """Copies of the blockset's storage: counts [R] int32 and cols [R, nB] int32
    (row r's first counts[r] entries are its ascending key-block ids)."""
    c, k = ctypes.c_void_p(), ctypes.c_void_p()
    _check(load_library().lbsa_blockset_views(bs.handle, ctypes.byref(c), ctypes.byref(k)))
    R = bs.B * bs.H * bs.nB
    counts = torch.as_tensor(_DeviceArray(c.value, R, "<i4"), device="cuda").clone()
    cols = torch.as_tensor(_DeviceArray(k.value, R * bs.nB, "<i4"), device="cuda").clone().view(R, bs.nB)
    return counts, cols


def lbsa_blockset_masks(bs: Blockset):
    """Copy of a per-token blockset's token sets, int64 [R, nB] (bit u of
    masks[r, t]: token u of row r's query block keeps its t-th listed key
    block), or None for blocksets of the other scopes."""
    m = ctypes.c_void_p()
    _check(load_library().lbsa_blockset_masks(bs.handle, ctypes.byref(m)))
    if not m.value:
        return None
    R = bs.B * bs.H * bs.nB
    return torch.as_tensor(_DeviceArray(m.value, R * bs.nB, "<i8"), device="cuda").clone().view(R, bs.nB)


def lbsa_score_attend(q, k, v, block: int, scores=None, out=None, lse=None, want_lse=False, stream=None):
    """Dense attention that also returns the exact block masses (one sweep).

    Returns (scores [B, H, nB, nB] fp32, out), or (scores, out, lse) when lse
    is asked for or given, as lbsa_score does."""
    _same_layout(q, k)
    _same_layout(q, v)
    B, H, N, _ = q.shape
    nB = -(-N // block)
    if scores is None:
        scores = torch.empty(B, H, nB, nB, dtype=torch.float32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    else:
        _same_layout(q, out)
    if want_lse and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    desc = _desc(q)
    _on_device(scores, "scores", torch.float32, B * H * nB * nB)
    _on_device(lse, "lse", torch.float32, B * H * N)
    _check(load_library().lbsa_score_attend(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(desc), block, _ptr(scores),
                                            _ptr(out), _ptr(lse), _stream(stream)))
    return (scores, out, lse) if (want_lse or lse is not None) else (scores, out)


_RULES = {"local_topk": 0, "topp_floor": 1}


def lbsa_select_rule(scores, block: int, rule: str, n_valid: int, p: float = 0.99, k: int = 0,
                     stream=None) -> Blockset:
    """Selection by a further rule into a new blockset (row scope): "local_topk"
    keeps each row's own key block plus the k top-ranked others; "topp_floor"
    applies the row threshold rule with p, then raises every row to its head's
    size-weighted mean count (rounded up)."""
    _on_device(scores, "scores")
    if scores.dtype != torch.float32 or not scores.is_contiguous() or scores.dim() != 4:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be a contiguous fp32 [B, H, nB, nB] tensor")
    B, H, nB, nB2 = scores.shape
    if nB != nB2:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be square per head")
    h = ctypes.c_void_p()
    _check(load_library().lbsa_select_rule(_ptr(scores), B, H, nB, block, int(n_valid), _RULES[rule], float(p),
                                           int(k), ctypes.byref(h), _stream(stream)))
    return Blockset(h.value)


def lbsa_select_routed(scores, block: int, p: float, entropy_threshold: float, group: int, stream=None):
    """Entropy-routed selection into a new blockset: heads whose normalised
    mean row entropy is below entropy_threshold are pooled, `group` at a time
    in head order, and each pool's rows of one query block compete together;
    the other heads take the row rule.  Returns (blockset, head entropy fp64
    [B, H], head domain int32 [B, H]: -1 per row, else the pool index)."""
    _on_device(scores, "scores")
    if scores.dtype != torch.float32 or not scores.is_contiguous() or scores.dim() != 4:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be a contiguous fp32 [B, H, nB, nB] tensor")
    B, H, nB, nB2 = scores.shape
    if nB != nB2:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be square per head")
    ent = torch.empty(B, H, dtype=torch.float64, device=scores.device)
    dom = torch.empty(B, H, dtype=torch.int32, device=scores.device)
    h = ctypes.c_void_p()
    _check(load_library().lbsa_select_routed(_ptr(scores), B, H, nB, block, float(p), float(entropy_threshold),
                                             int(group), _ptr(ent), _ptr(dom), ctypes.byref(h), _stream(stream)))
    return Blockset(h.value), ent, dom


def lbsa_attend(q, k, v, bs: Blockset, out=None, lse=None, want_lse=False, stream=None):
    """Block-sparse attention of q over the kept blocks of bs; returns out (and lse)."""
    _same_layout(q, k)
    _same_layout(q, v)
    if out is None:
        out = torch.empty_like(q)
    else:
        _same_layout(q, out)
    if want_lse and lse is None:
        lse = torch.empty(q.shape[0], q.shape[1], q.shape[2], dtype=torch.float32, device=q.device)
    desc = _desc(q)
    _on_device(lse, "lse", torch.float32, q.shape[0] * q.shape[1] * q.shape[2])
    _check(load_library().lbsa_attend(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(desc), bs.handle,
                                      _ptr(out), _ptr(lse), _stream(stream)))
    return (out, lse) if (want_lse or lse is not None) else out


def lbsa_free(bs: Blockset):
    bs.free()


def lbsa_blockset_info(bs: Blockset) -> dict:
    return {"B": bs.B, "H": bs.H, "nB": bs.nB, "block": bs.block, "scope": bs.scope}


def lbsa_blockset_export(bs: Blockset, stream=None):
    """Compact CSR (row_ptr [R+1], col [nnz]) as int32 device tensors."""
    R = bs.B * bs.H * bs.nB
    dev = torch.device("cuda", torch.cuda.current_device())
    row_ptr = torch.empty(R + 1, dtype=torch.int32, device=dev)
    col = torch.empty(max(R * bs.nB, 1), dtype=torch.int32, device=dev)
    nnz = ctypes.c_int64()
    _check(load_library().lbsa_blockset_export(bs.handle, _ptr(row_ptr), _ptr(col), ctypes.byref(nnz),
                                               _stream(stream)))
    return row_ptr, col[:nnz.value]


def lbsa_blockset_from_csr(row_ptr, col, B: int, H: int, nB: int, block: int, stream=None) -> Blockset:
    """Blockset from a CSR on the device (row_ptr [B*H*nB + 1], col [nnz]).  The
    row pointers are checked here (start at 0, never decrease, end inside col),
    since the library indexes col with them; column ids are checked on the
    device (status word)."""
    _on_device(row_ptr, "row_ptr", contiguous=False)
    _on_device(col, "col", contiguous=False)
    row_ptr = row_ptr.to(torch.int32).contiguous()
    col = col.to(torch.int32).contiguous()
    R = B * H * nB
    if row_ptr.numel() != R + 1:
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"row_ptr holds {row_ptr.numel()} entries, B*H*nB + 1 = {R + 1} needed")
    rp = row_ptr.cpu()
    if int(rp[0]) != 0 or bool((rp[1:] < rp[:-1]).any()) or int(rp[-1]) > col.numel():
        raise LbsaError(LBSA_ERR_INVALID_ARG, "row_ptr must start at 0, never decrease and end within col")
    if col.numel() == 0:
        col = torch.zeros(1, dtype=torch.int32, device=row_ptr.device)
    h = ctypes.c_void_p()
    _check(load_library().lbsa_blockset_from_csr(_ptr(row_ptr), _ptr(col), B, H, nB, block,
                                                 ctypes.byref(h), _stream(stream)))
    return Blockset(h.value, keep=(row_ptr, col))


def lbsa_blockset_export_bitmask(bs: Blockset, stream=None):
    """The blockset as a block bitmask: int32 [B, H, nB, ceil(nB/32)] on the
    device (the bits of uint32 words), bit j % 32 of word j // 32 of a row set
    when key block j is kept."""
    W = (bs.nB + 31) // 32
    bits = torch.empty(bs.B, bs.H, bs.nB, W, dtype=torch.int32, device=torch.device("cuda", torch.cuda.current_device()))
    _check(load_library().lbsa_blockset_export_bitmask(bs.handle, _ptr(bits), _stream(stream)))
    return bits


def lbsa_blockset_from_bitmask(bits, block: int, stream=None) -> Blockset:
    """Blockset from a block bitmask on the device, int32 (or uint32 bits)
    [B, H, nB, ceil(nB/32)] in the layout lbsa_blockset_export_bitmask writes."""
    if bits.dim() != 4:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "bits must be [B, H, nB, ceil(nB/32)]")
    B, H, nB, W = bits.shape
    if W != (nB + 31) // 32:
        raise LbsaError(LBSA_ERR_INVALID_ARG, f"{W} words a row, ceil(nB/32) = {(nB + 31) // 32} needed")
    if bits.dtype not in (torch.int32, torch.uint32):
        raise LbsaError(LBSA_ERR_INVALID_ARG, "bits must be int32 or uint32")
    _on_device(bits, "bits", bits.dtype, B * H * nB * W)
    h = ctypes.c_void_p()
    _check(load_library().lbsa_blockset_from_bitmask(_ptr(bits), B, H, nB, block, ctypes.byref(h), _stream(stream)))
    return Blockset(h.value, keep=(bits,))


def lbsa_get_status(bs: Blockset, clear: bool = False, stream=None) -> int:
    st = ctypes.c_int32()
    _check(load_library().lbsa_get_status(bs.handle, ctypes.byref(st), int(clear), _stream(stream)))
    return st.value


def lbsa_device_status(clear: bool = False, stream=None) -> int:
    st = ctypes.c_int32()
    _check(load_library().lbsa_device_status(ctypes.byref(st), int(clear), _stream(stream)))
    return st.value


def lbsa_partition_perm(T: int, H: int, W: int, kind: str, tile=(4, 4, 4), frame_tile=(8, 8),
                        device=None, stream=None):
    """Token order of a (T, H, W) grid: blocked[slot] = raster[perm[slot]] (int32).

    device=None fills a host tensor on the CPU (library host code); a CUDA
    device fills a device tensor with the library's kernel.
    """
    k = _PARTS[kind]
    tt, th, tw = tile if kind == "3d" else (1, *frame_tile) if kind == "2d" else (1, 1, 1)
    n = T * H * W
    lib = load_library()
    if device is None:
        perm = torch.empty(n, dtype=torch.int32)
        _check(lib.lbsa_partition_perm(T, H, W, k, tt, th, tw, _ptr(perm), 0, None))
    else:
        perm = torch.empty(n, dtype=torch.int32, device=device)
        _check(lib.lbsa_partition_perm(T, H, W, k, tt, th, tw, _ptr(perm), 1, _stream(stream)))
    return perm


def lbsa_permute(xs, perm, inverse: bool = False, outs=None, stream=None):
    """Gather (inverse=False: y[slot] = x[perm[slot]]) or scatter rows of 1..3 tensors."""
    xs = list(xs)
    for x in xs[1:]:
        _same_layout(xs[0], x)
    outs = [torch.empty_like(x) for x in xs] if outs is None else list(outs)
    for o in outs:
        _same_layout(xs[0], o)
    desc = _desc(xs[0])
    # entries outside [0, N) are skipped by the kernel and reported in the device status word
    _on_device(perm, "perm", torch.int32, xs[0].shape[2])
    n = len(xs)
    xa = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
    ya = (ctypes.c_void_p * n)(*[y.data_ptr() for y in outs])
    _check(load_library().lbsa_permute(xa, ya, n, _ptr(perm), ctypes.byref(desc), int(inverse),
                                       _stream(stream)))
    return outs


def lbsa_selftest_wait(limit_us: int = 1000, stream=None) -> int:
    """Run the bounded-wait self test; returns the device status it reported."""
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(load_library().lbsa_selftest_wait(limit_us, _ptr(out), _stream(stream)))
    return int(out.item())


def lbsa_selftest_exp2(v, stream=None):
    """2^v through the scorer's FMA-pipe exponential (float32 CUDA tensor)."""
    if v.dtype != torch.float32 or not v.is_cuda:
        raise TypeError("v must be a float32 CUDA tensor")
    v = v.contiguous()
    out = torch.empty_like(v)
    _check(load_library().lbsa_selftest_exp2(_ptr(v), _ptr(out), v.numel(), _stream(stream)))
    return out


def lbsa_select_head_noalloc(scores, p: float, counts=None, cols=None, status=None, stream=None):
    """Head-scope selection into caller buffers; the library allocates nothing.

    Returns (counts [B*H*nB], cols [B*H*nB*nB], status [1]) int32 device
    tensors; row r's kept ids are cols[r*nB : r*nB + counts[r]].
    """
    _on_device(scores, "scores", torch.float32)
    if scores.dim() != 4 or scores.shape[2] != scores.shape[3]:
        raise LbsaError(LBSA_ERR_INVALID_ARG, "scores must be [B, H, nB, nB]")
    B, H, nB, _ = scores.shape
    dev = scores.device
    counts = torch.empty(B * H * nB, dtype=torch.int32, device=dev) if counts is None else counts
    cols = torch.empty(B * H * nB * nB, dtype=torch.int32, device=dev) if cols is None else cols
    status = torch.empty(1, dtype=torch.int32, device=dev) if status is None else status
    _on_device(counts, "counts", torch.int32, B * H * nB)
    _on_device(cols, "cols", torch.int32, B * H * nB * nB)
    _on_device(status, "status", torch.int32, 1)
    _check(load_library().lbsa_select_head_noalloc(_ptr(scores), B, H, nB, float(p), _ptr(counts), _ptr(cols),
                                                   _ptr(status), _stream(stream)))
    return counts, cols, status


def lbsa_last_error() -> str:
    return load_library().lbsa_last_error().decode()


def lbsa_version() -> int:
    return load_library().lbsa_version()
