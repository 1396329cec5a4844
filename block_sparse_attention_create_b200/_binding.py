"""ctypes binding of libfa.so, the B200 block-sparse attention library.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  The C-ABI names are re-exported unchanged (``fa_create_block_mask``,
``fa_flex_attention_fwd``, ...); ``create_block_mask`` and ``flex_attention`` are
thin conveniences that allocate the output tensors with torch and pass pointers,
mirroring the FlexAttention calls of the how-to
("FlexAttention on Apple Silicon: block mask how-to", dreaming.press, "Setup").

There is no fallback: if libfa.so is missing or cannot be loaded, importing this
module raises ImportError.  Build it with
``python -m block_sparse_attention_create_b200.build``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

(FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT,
 FA_ERR_SCRATCH_TOO_SMALL) = range(6)
FA_MASK_CAUSAL, FA_MASK_SLIDING_WINDOW_CAUSAL, FA_MASK_DOCUMENT_CAUSAL, FA_MASK_BITMAP = range(4)
FA_SCORE_NONE, FA_SCORE_TANH_SOFTCAP = range(2)
FA_BF16, FA_FP16 = range(2)
FA_DECODE_FULL, FA_DECODE_CAUSAL, FA_DECODE_SLIDING_WINDOW = range(3)
FA_DECODE_MAX_ROWS = 32
FA_BLOCK = 128
FA_MAX_LEN = 8192 * 128
FA_NOALLOC_SCRATCH_BYTES = 4 << 20

# Every symbol include/fa.h declares.
EXPORTED = ("fa_block_mask_dims", "fa_create_block_mask", "fa_fwd_workspace_bytes",
            "fa_flex_attention_fwd", "fa_get_last_device_error", "fa_status_string",
            "fa_num_sms", "fa_flex_attention_fwd_noalloc", "fa_create_block_mask_bitmap",
            "fa_block_mask_transpose", "fa_flex_attention_fwd_gqa", "fa_decode_workspace_bytes",
            "fa_flex_attention_decode", "fa_debug_set_mma_stall", "fa_create_block_mask_bh",
            "fa_bwd_workspace_bytes", "fa_flex_attention_bwd", "fa_block_mask_validate")


class fa_block_mask(ctypes.Structure):
    """Mirror of ``struct fa_block_mask`` in include/fa.h."""
    _fields_ = [
        ("kv_num_blocks", ctypes.c_void_p),
        ("kv_indices", ctypes.c_void_p),
        ("full_kv_num_blocks", ctypes.c_void_p),
        ("full_kv_indices", ctypes.c_void_p),
        ("q_order", ctypes.c_void_p),
        ("q_len", ctypes.c_int32),
        ("kv_len", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("n_q_blocks", ctypes.c_int32),
        ("n_kv_blocks", ctypes.c_int32),
        ("kind", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("doc_id", ctypes.c_void_p),
        ("bitmap", ctypes.c_void_p),
        ("mask_batch", ctypes.c_int32),
        ("mask_heads", ctypes.c_int32),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_attention_create_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i32, vp, f32 = ctypes.c_int32, ctypes.c_void_p, ctypes.c_float
    lib.fa_block_mask_dims.argtypes = [i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.fa_block_mask_dims.restype = i32
    lib.fa_create_block_mask.argtypes = [i32, i32, vp, i32, i32, i32, ctypes.POINTER(fa_block_mask), vp]
    lib.fa_create_block_mask.restype = i32
    lib.fa_fwd_workspace_bytes.argtypes = []
    lib.fa_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_flex_attention_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                          ctypes.POINTER(fa_block_mask), i32, f32, f32, vp, vp, vp, vp]
    lib.fa_flex_attention_fwd.restype = i32
    lib.fa_get_last_device_error.argtypes = [vp, vp]
    lib.fa_get_last_device_error.restype = i32
    lib.fa_status_string.argtypes = [i32]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_num_sms.argtypes = []
    lib.fa_num_sms.restype = i32
    lib.fa_flex_attention_fwd_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                  i32, i32, vp, i32, f32, f32, vp, vp, vp, vp]
    lib.fa_flex_attention_fwd_noalloc.restype = i32
    lib.fa_create_block_mask_bitmap.argtypes = [vp, i32, i32, i32, ctypes.POINTER(fa_block_mask), vp]
    lib.fa_create_block_mask_bitmap.restype = i32
    lib.fa_block_mask_transpose.argtypes = [ctypes.POINTER(fa_block_mask), vp, vp, vp, vp, vp]
    lib.fa_block_mask_transpose.restype = i32
    lib.fa_flex_attention_fwd_gqa.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                              ctypes.POINTER(fa_block_mask), i32, f32, f32, vp, vp,
                                              vp, vp]
    lib.fa_flex_attention_fwd_gqa.restype = i32
    lib.fa_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.fa_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_flex_attention_decode.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                             i32, i32, f32, f32, vp, vp, vp, ctypes.c_size_t, vp]
    lib.fa_flex_attention_decode.restype = i32
    lib.fa_debug_set_mma_stall.argtypes = [i32, ctypes.c_uint64]
    lib.fa_debug_set_mma_stall.restype = None
    lib.fa_create_block_mask_bh.argtypes = [i32, i32, vp, vp, i32, i32, i32, i32, i32,
                                            ctypes.POINTER(fa_block_mask), vp]
    lib.fa_create_block_mask_bh.restype = i32
    lib.fa_bwd_workspace_bytes.argtypes = [i32, i32, i32]
    lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_flex_attention_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                          ctypes.POINTER(fa_block_mask), vp, vp, vp, vp, i32, f32,
                                          f32, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.fa_flex_attention_bwd.restype = i32
    lib.fa_block_mask_validate.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32,
                                           ctypes.POINTER(ctypes.c_int64)]
    lib.fa_block_mask_validate.restype = i32
    return lib


_lib = _load()

# ---- the C-ABI, same names --------------------------------------------------
fa_block_mask_dims = _lib.fa_block_mask_dims
fa_create_block_mask = _lib.fa_create_block_mask
fa_fwd_workspace_bytes = _lib.fa_fwd_workspace_bytes
fa_flex_attention_fwd = _lib.fa_flex_attention_fwd
fa_get_last_device_error = _lib.fa_get_last_device_error
fa_status_string = _lib.fa_status_string
fa_num_sms = _lib.fa_num_sms
fa_flex_attention_fwd_noalloc = _lib.fa_flex_attention_fwd_noalloc
fa_create_block_mask_bitmap = _lib.fa_create_block_mask_bitmap
fa_block_mask_transpose = _lib.fa_block_mask_transpose
fa_flex_attention_fwd_gqa = _lib.fa_flex_attention_fwd_gqa
fa_decode_workspace_bytes = _lib.fa_decode_workspace_bytes
fa_flex_attention_decode = _lib.fa_flex_attention_decode
fa_debug_set_mma_stall = _lib.fa_debug_set_mma_stall
fa_create_block_mask_bh = _lib.fa_create_block_mask_bh
fa_bwd_workspace_bytes = _lib.fa_bwd_workspace_bytes
fa_flex_attention_bwd = _lib.fa_flex_attention_bwd
fa_block_mask_validate = _lib.fa_block_mask_validate


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {fa_status_string(status).decode()}")


def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def block_mask_dims(q_len: int, kv_len: int, block: int = FA_BLOCK):
    nq, nkv = ctypes.c_int32(), ctypes.c_int32()
    _check(fa_block_mask_dims(q_len, kv_len, block, ctypes.byref(nq), ctypes.byref(nkv)),
           "fa_block_mask_dims")
    return nq.value, nkv.value


class BlockMask:
    """Device block tables of one mask (broadcast over batch and heads).

    Holds the torch tensors the library fills and the ctypes struct that points
    at them; reuse one BlockMask across forwards, as the how-to recommends.
    """

    def __init__(self, q_len: int, kv_len: int, device, block: int = FA_BLOCK,
                 mask_batch: int = 1, mask_heads: int = 1):
        nq, nkv = block_mask_dims(q_len, kv_len, block)
        inst = mask_batch * mask_heads   # per-(batch, head) instances, instance-major
        i32 = dict(dtype=torch.int32, device=device)
        self.kv_num_blocks = torch.zeros(inst * nq, **i32)
        self.kv_indices = torch.zeros(inst * nq, nkv, **i32)
        self.full_kv_num_blocks = torch.zeros(inst * nq, **i32)
        self.full_kv_indices = torch.zeros(inst * nq, nkv, **i32)
        self.q_order = torch.zeros(inst * 2 * nq, **i32)   # schedule: (row, partial | full << 16)
        self.mask_batch, self.mask_heads = mask_batch, mask_heads
        self.doc_id: Optional[torch.Tensor] = None
        self.bitmap: Optional[torch.Tensor] = None
        self.struct = fa_block_mask()
        self.struct.kv_num_blocks = self.kv_num_blocks.data_ptr()
        self.struct.kv_indices = self.kv_indices.data_ptr()
        self.struct.full_kv_num_blocks = self.full_kv_num_blocks.data_ptr()
        self.struct.full_kv_indices = self.full_kv_indices.data_ptr()
        self.struct.q_order = self.q_order.data_ptr()
        self.q_len, self.kv_len, self.n_q_blocks, self.n_kv_blocks = q_len, kv_len, nq, nkv

    def tables(self):
        """Host copies of the integer tables (for inspection and tests)."""
        return {k: getattr(self, k).cpu().numpy() for k in
                ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices", "q_order")}

    def validate(self):
        """fa_block_mask_validate on host copies of the tables (synchronises).
        Returns (status, first offending instance * nQ + row or -1)."""
        return validate_tables(self.tables(), self.n_q_blocks, self.n_kv_blocks,
                               self.mask_batch * self.mask_heads)

    def transpose(self, stream: Optional[torch.cuda.Stream] = None):
        """fa_block_mask_transpose: per kv block, its partial / full q blocks (device
        tensors q_num_blocks [nKV], q_indices [nKV, nQ], full_q_num_blocks,
        full_q_indices)."""
        nq, nkv = self.n_q_blocks, self.n_kv_blocks
        inst = self.mask_batch * self.mask_heads
        i32 = dict(dtype=torch.int32, device=self.kv_num_blocks.device)
        t = {"q_num_blocks": torch.zeros(inst * nkv, **i32),
             "q_indices": torch.zeros(inst * nkv, nq, **i32),
             "full_q_num_blocks": torch.zeros(inst * nkv, **i32),
             "full_q_indices": torch.zeros(inst * nkv, nq, **i32)}
        _check(fa_block_mask_transpose(ctypes.byref(self.struct), _ptr(t["q_num_blocks"]),
                                       _ptr(t["q_indices"]), _ptr(t["full_q_num_blocks"]),
                                       _ptr(t["full_q_indices"]), _stream_handle(stream)),
               "fa_block_mask_transpose")
        return t


def validate_tables(tables: dict, n_q_blocks: int, n_kv_blocks: int, instances: int = 1):
    """fa_block_mask_validate on host (numpy) tables: keys kv_num_blocks, kv_indices,
    full_kv_num_blocks, full_kv_indices, q_order (as BlockMask.tables() returns them).
    Returns (status, first offending instance * nQ + row, or -1)."""
    import numpy as np
    arrs = [np.ascontiguousarray(tables[k], dtype=np.int32) for k in
            ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices", "q_order")]
    bad = ctypes.c_int64(0)
    st = fa_block_mask_validate(*(ctypes.c_void_p(a.ctypes.data) for a in arrs), n_q_blocks,
                                n_kv_blocks, instances, ctypes.byref(bad))
    return st, bad.value


def create_block_mask(kind: int, q_len: int, kv_len: int, window: int = 0,
                      doc_id: Optional[torch.Tensor] = None, device="cuda",
                      stream: Optional[torch.cuda.Stream] = None, out: Optional[BlockMask] = None,
                      bitmap: Optional[torch.Tensor] = None, B: Optional[int] = None,
                      H: Optional[int] = None) -> BlockMask:
    """fa_create_block_mask (or, for FA_MASK_BITMAP, fa_create_block_mask_bitmap with
    `bitmap`: an int32 CUDA tensor (q_len, 4 * nKV) holding the 32-bit words) on fresh
    (or the given) device tables.  With B and / or H (the how-to's create_block_mask
    arguments), one mask per batch element / head: fa_create_block_mask_bh, with
    doc_id (instances, max(q_len, kv_len)) or bitmap (instances, q_len, 4 * nKV)."""
    mb, mh = (B or 1), (H or 1)
    if mb > 1 or mh > 1:
        bm = out if out is not None else BlockMask(q_len, kv_len, device, mask_batch=mb,
                                                   mask_heads=mh)
        n = max(q_len, kv_len)
        if doc_id is not None:
            if (doc_id.dtype != torch.int32 or not doc_id.is_cuda or not doc_id.is_contiguous()
                    or doc_id.numel() < mb * mh * n):
                raise ValueError("doc_id must be a contiguous int32 CUDA tensor (B*H, max(L, S))")
            bm.doc_id = doc_id
        if bitmap is not None:
            if (bitmap.dtype != torch.int32 or not bitmap.is_cuda or not bitmap.is_contiguous()
                    or bitmap.numel() != mb * mh * q_len * 4 * bm.n_kv_blocks):
                raise ValueError("bitmap must be a contiguous int32 CUDA tensor "
                                 "(B*H, q_len, 4 * nKV)")
            bm.bitmap = bitmap
        _check(fa_create_block_mask_bh(kind, window, _ptr(doc_id), _ptr(bitmap), mb, mh, q_len,
                                       kv_len, FA_BLOCK, ctypes.byref(bm.struct),
                                       _stream_handle(stream)),
               "fa_create_block_mask_bh")
        return bm
    bm = out if out is not None else BlockMask(q_len, kv_len, device)
    if kind == FA_MASK_BITMAP:
        if (bitmap is None or bitmap.dtype != torch.int32 or not bitmap.is_cuda
                or not bitmap.is_contiguous() or bitmap.shape != (q_len, 4 * bm.n_kv_blocks)):
            raise ValueError("bitmap must be a contiguous int32 CUDA tensor (q_len, 4 * nKV)")
        bm.bitmap = bitmap
        _check(fa_create_block_mask_bitmap(_ptr(bitmap), q_len, kv_len, FA_BLOCK,
                                           ctypes.byref(bm.struct), _stream_handle(stream)),
               "fa_create_block_mask_bitmap")
        return bm
    if doc_id is not None:
        if doc_id.dtype != torch.int32 or not doc_id.is_cuda or not doc_id.is_contiguous():
            raise ValueError("doc_id must be a contiguous int32 CUDA tensor")
        if doc_id.numel() < max(q_len, kv_len):
            raise ValueError("doc_id must hold max(q_len, kv_len) ids")
        bm.doc_id = doc_id
    _check(fa_create_block_mask(kind, window, _ptr(doc_id), q_len, kv_len, FA_BLOCK,
                                ctypes.byref(bm.struct), _stream_handle(stream)),
           "fa_create_block_mask")
    return bm


_workspaces = {}


def workspace(device) -> torch.Tensor:
    """A zeroed forward workspace per device (reused by every call on that device)."""
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros(int(fa_fwd_workspace_bytes()), dtype=torch.uint8, device=f"cuda:{key}")
        _workspaces[key] = ws
    return ws


_DTYPES = {torch.bfloat16: FA_BF16, torch.float16: FA_FP16}


def flex_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_mask: BlockMask,
                   score_mod: int = FA_SCORE_NONE, softcap: float = 0.0, scale: float = 0.0,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   return_lse: bool = False, ws: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None):
    """fa_flex_attention_fwd on torch tensors q (B,H,L,D), k/v (B,H,S,D); with k/v
    (B,Hkv,S,D), Hkv < H dividing H, fa_flex_attention_fwd_gqa."""
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype bf16 or fp16")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k, v must be contiguous 4-D CUDA tensors")
    B, H, L, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, S, D) or v.shape != (B, Hkv, S, D) or Hkv < 1 or H % Hkv:
        raise ValueError("k and v must be (B, Hkv, S, D) with the q's B and D, Hkv dividing H")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(B, H, L, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(q.device)
    if Hkv == H:
        _check(fa_flex_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], B, H, L, S, D,
                                     ctypes.byref(block_mask.struct), score_mod, float(softcap),
                                     float(scale), _ptr(out), _ptr(lse), _ptr(ws),
                                     _stream_handle(stream)),
               "fa_flex_attention_fwd")
    else:
        _check(fa_flex_attention_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], B, H, Hkv, L,
                                         S, D, ctypes.byref(block_mask.struct), score_mod,
                                         float(softcap), float(scale), _ptr(out), _ptr(lse),
                                         _ptr(ws), _stream_handle(stream)),
               "fa_flex_attention_fwd_gqa")
    return (out, lse) if return_lse else out


def flex_attention_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask_kind: int,
                           window: int = 0, doc_id: Optional[torch.Tensor] = None,
                           score_mod: int = FA_SCORE_NONE, softcap: float = 0.0,
                           scale: float = 0.0, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None,
                           device_error: Optional[torch.Tensor] = None, check: bool = False,
                           stream: Optional[torch.cuda.Stream] = None):
    """fa_flex_attention_fwd_noalloc: mask build + forward with the library's static
    scratch (no block tables or workspace from the caller).

    q (B,H,L,D), k / v (B,H,S,D) share dtype and device.  `out` (B,H,L,D, q's dtype),
    `lse` (B,H,L float32) and `device_error` (int32, at least one element) belong to
    the caller; any that is not given is created here with torch (so this
    convenience allocates; the C entry point itself does not).  The device error
    word is copied into `device_error` in stream order: nonzero means a bounded
    device wait gave up and the outputs are invalid.  With `check`, the stream is
    synchronised and a nonzero word raises FAError(FA_ERR_TIMEOUT); without it,
    the caller reads `device_error` when it likes.  Returns (out, lse)."""
    # shapes and dtypes first, then devices (so each mistake gets its own message)
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype bf16 or fp16")
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    B, H, L, D = q.shape
    S = k.shape[2]
    if k.shape != (B, H, S, D) or v.shape != (B, H, S, D):
        raise ValueError("k and v must be (B, H, S, D) with the q's B, H and D")
    if mask_kind == FA_MASK_DOCUMENT_CAUSAL and (
            doc_id is None or doc_id.dtype != torch.int32 or doc_id.numel() < max(L, S)):
        raise ValueError("doc_id must be an int32 tensor of max(L, S) ids")
    if out is not None and (out.shape != q.shape or out.dtype != q.dtype):
        raise ValueError("out must have q's shape and dtype")
    if lse is not None and (lse.shape != (B, H, L) or lse.dtype != torch.float32):
        raise ValueError("lse must be a float32 (B, H, L) tensor")
    if device_error is not None and (device_error.dtype != torch.int32
                                     or device_error.numel() < 1):
        raise ValueError("device_error must be an int32 tensor of at least one element")
    given = [t for t in (q, k, v, doc_id, out, lse, device_error) if t is not None]
    if any(not t.is_cuda or t.device != q.device or not t.is_contiguous() for t in given):
        raise ValueError("every tensor must be a contiguous CUDA tensor on q's device")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, H, L, dtype=torch.float32, device=q.device)
    if device_error is None:
        device_error = torch.zeros(1, dtype=torch.int32, device=q.device)
    # the scratch is the current device's: make q's device current for the call
    with torch.cuda.device(q.device):
        _check(fa_flex_attention_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], B, H, L,
                                             S, D, mask_kind, window, _ptr(doc_id), score_mod,
                                             float(softcap), float(scale), _ptr(out), _ptr(lse),
                                             _ptr(device_error), _stream_handle(stream)),
               "fa_flex_attention_fwd_noalloc")
        if check:
            (stream if stream is not None else torch.cuda.current_stream()).synchronize()
            if int(device_error.reshape(-1)[0].item()) != 0:
                raise FAError(FA_ERR_TIMEOUT, "fa_flex_attention_fwd_noalloc")
    return out, lse


_decode_workspaces = {}


def decode_workspace(device, nbytes: int) -> torch.Tensor:
    """A zeroed decode workspace of at least `nbytes` per device (grown on demand)."""
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    ws = _decode_workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=f"cuda:{key}")
        _decode_workspaces[key] = ws
    return ws


def flex_attention_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          mask: int = FA_DECODE_CAUSAL, window: int = 0,
                          score_mod: int = FA_SCORE_NONE, softcap: float = 0.0, scale: float = 0.0,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                          return_lse: bool = False, ws: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None):
    """fa_flex_attention_decode: q (B,H,L,D) new queries against the cache k/v
    (B,Hkv,S,D), lower-right aligned."""
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype bf16 or fp16")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k, v must be contiguous 4-D CUDA tensors")
    B, H, L, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, S, D) or v.shape != (B, Hkv, S, D) or Hkv < 1 or H % Hkv:
        raise ValueError("k and v must be (B, Hkv, S, D) with the q's B and D, Hkv dividing H")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(B, H, L, dtype=torch.float32, device=q.device)
    need = int(fa_decode_workspace_bytes(B, H, Hkv, L, S, D))
    if ws is None:
        ws = decode_workspace(q.device, need)
    _check(fa_flex_attention_decode(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], B, H, Hkv, L, S, D,
                                    mask, window, score_mod, float(softcap), float(scale),
                                    _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                    _stream_handle(stream)),
           "fa_flex_attention_decode")
    return (out, lse) if return_lse else out


def flex_attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                            dout: torch.Tensor, lse: torch.Tensor, block_mask: BlockMask,
                            score_mod: int = FA_SCORE_NONE, softcap: float = 0.0,
                            scale: float = 0.0, columns: Optional[dict] = None,
                            check: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """fa_flex_attention_bwd: (dq, dk, dv) of the forward that produced out and lse.
    `columns`: the mask's column lists (block_mask.transpose()); built here if None.
    With `check`, the stream is synchronised and a bounded device wait that gave up
    raises FAError(FA_ERR_TIMEOUT)."""
    for t in (q, k, v, out, dout):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype != q.dtype:
            raise ValueError("q, k, v, out, dout must be contiguous 4-D CUDA tensors of one dtype")
    if q.dtype not in _DTYPES:
        raise ValueError("dtype must be bf16 or fp16")
    B, H, L, D = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, S, D) or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("shape mismatch")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (B, H, L):
        raise ValueError("lse must be a contiguous float32 (B, H, L) tensor")
    cols = columns if columns is not None else block_mask.transpose(stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = int(fa_bwd_workspace_bytes(B, H, L))
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    ws[:256].zero_()  # the device error word
    _check(fa_flex_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                 _DTYPES[q.dtype], B, H, Hkv, L, S, D,
                                 ctypes.byref(block_mask.struct), _ptr(cols["q_num_blocks"]),
                                 _ptr(cols["q_indices"]), _ptr(cols["full_q_num_blocks"]),
                                 _ptr(cols["full_q_indices"]), score_mod, float(softcap),
                                 float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                 _stream_handle(stream)),
           "fa_flex_attention_bwd")
    if check:
        _check(fa_get_last_device_error(_ptr(ws), _stream_handle(stream)), "fa_flex_attention_bwd")
    return dq, dk, dv


def last_decode_error(device=None, stream: Optional[torch.cuda.Stream] = None) -> int:
    """fa_get_last_device_error on the per-device decode workspace."""
    dev = device if device is not None else torch.cuda.current_device()
    return fa_get_last_device_error(_ptr(decode_workspace(dev, 256)), _stream_handle(stream))


def last_device_error(device=None, stream: Optional[torch.cuda.Stream] = None) -> int:
    """fa_get_last_device_error on the per-device workspace; returns the status."""
    dev = device if device is not None else torch.cuda.current_device()
    return fa_get_last_device_error(_ptr(workspace(dev)), _stream_handle(stream))


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
