"""ctypes binding of libkvq (include/kvq.h): argument marshalling only.

Every function here forwards to the C entry point of the same name. Torch tensors are
used for device memory and the current CUDA stream; all computation happens in the
library's CUDA kernels. If libkvq.so is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK = 0
STATUS_NAMES = ["OK", "ERR_ARG", "ERR_SHAPE", "ERR_DTYPE", "ERR_BUDGET", "ERR_RANGE", "ERR_WORKSPACE",
                "ERR_CUDA", "ERR_TIMEOUT", "ERR_UNSUPPORTED", "ERR_MISMATCH"]
KVQ_ERR_TIMEOUT = 8
KVQ_ERR_MISMATCH = 10
KVQ_F32, KVQ_F16, KVQ_BF16 = 0, 1, 2
MODE_BLOCKGTQ, MODE_UNIFORM = 0, 1
TILE = 32
HEAD_DIM = 128


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        detail = ""
        if status == 7 and _lib is not None:
            detail = f" [{_lib.kvq_last_cuda_error().decode()}]"
        super().__init__(f"{fn} failed: KVQ_{name} ({status}){detail}")
        self.status = status


class Tensor4(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64),
                ("stride_t", ctypes.c_int64), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class CalibParams(ctypes.Structure):
    _fields_ = [("bits_k", ctypes.c_int32), ("w_max", ctypes.c_int32), ("n_calib", ctypes.c_int32),
                ("mode", ctypes.c_int32)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("bits_k", ctypes.c_int32), ("bits_v", ctypes.c_int32)]


class HeadAlloc(ctypes.Structure):
    _fields_ = [("energy", ctypes.c_double * 64), ("gain", ctypes.c_float * 64), ("dequant", ctypes.c_float * 64),
                ("bit_off", ctypes.c_int16 * 64), ("width", ctypes.c_uint8 * 64),
                ("stream_block", ctypes.c_uint8 * 64), ("class_bit", ctypes.c_uint16 * 8),
                ("class_width", ctypes.c_uint8 * 8), ("class_first", ctypes.c_uint8 * 8),
                ("class_blocks", ctypes.c_uint8 * 8), ("reserved_b", ctypes.c_uint8 * 56),
                ("head_dim", ctypes.c_int32), ("bits_k", ctypes.c_int32), ("w_max", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("n_classes", ctypes.c_int32), ("k_words", ctypes.c_int32),
                ("n_blocks", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("plan_slot", ctypes.c_uint32 * 24), ("plan_col_block", ctypes.c_int8 * 96),
                ("plan_n_slots", ctypes.c_int32), ("plan_k_cols", ctypes.c_int32), ("digest", ctypes.c_uint64),
                ("reserved_c", ctypes.c_uint8 * 432)]


class PackedHeader(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("layout_version", ctypes.c_uint16), ("head_dim", ctypes.c_uint16),
                ("bits_k", ctypes.c_uint8), ("bits_v", ctypes.c_uint8), ("w_max", ctypes.c_uint8),
                ("mode", ctypes.c_uint8), ("status", ctypes.c_uint32), ("batch", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("capacity", ctypes.c_int32), ("record_bytes", ctypes.c_uint32),
                ("reserved", ctypes.c_uint8 * 32)]


class DecodeExtra(ctypes.Structure):
    _fields_ = [("V", ctypes.c_void_p), ("vd", Tensor4), ("K_recent", ctypes.c_void_p), ("krd", Tensor4),
                ("V_recent", ctypes.c_void_p), ("vrd", Tensor4)]


_VP = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I = ctypes.c_int
_P4 = ctypes.POINTER(Tensor4)
_PC = ctypes.POINTER(CacheDesc)

_SIGNATURES = {
    "kvq_abi_version": ([], _I),
    "kvq_status_string": ([_I], ctypes.c_char_p),
    "kvq_codebook": ([_I, _VP, _VP, _VP], _I),
    "kvq_nf4_table": ([_VP, _VP], _I),
    "kvq_alloc_bytes": ([_I], _SZ),
    "kvq_calibrate_workspace_bytes": ([_I, _I, _I], _SZ),
    "kvq_packed_bytes": ([_PC], _SZ),
    "kvq_packed_header_bytes": ([_I], _SZ),
    "kvq_packed_status": ([_VP, _VP, ctypes.POINTER(_I)], _I),
    "kvq_debug_decode": ([_I, _I], _I),
    "kvq_last_cuda_error": ([], ctypes.c_char_p),
    "kvq_decode_workspace_bytes": ([_PC, _I], _SZ),
    "kvq_init": ([], _I),
    "kvq_workspace_init": ([_VP, _SZ, _VP], _I),
    "kvq_workspace_status": ([_VP, _VP, ctypes.POINTER(_I)], _I),
    "kvq_calibrate": ([_VP, _P4, ctypes.POINTER(CalibParams), _VP, _VP, _SZ, _VP], _I),
    "kvq_quantize": ([_VP, _P4, _VP, _P4, _VP, _PC, _VP, _VP], _I),
    "kvq_append": ([_VP, _P4, _VP, _P4, _VP, _PC, _I, _VP, _VP], _I),
    "kvq_decode_attn": ([_VP, _P4, _VP, _VP, _PC, _I, _VP, _VP, _SZ, _VP], _I),
    "kvq_decode_attn_ex": ([_VP, _P4, _VP, _VP, _PC, _I, ctypes.POINTER(DecodeExtra), _VP, _VP, _SZ, _VP], _I),
    "kvq_nf4_packed_bytes": ([_I, _I, _I, _I], _SZ),
    "kvq_nf4_decode_workspace_bytes": ([_I, _I, _I, _I], _SZ),
    "kvq_nf4_quantize": ([_VP, _P4, _VP, _P4, _I, _VP, _VP], _I),
    "kvq_nf4_append": ([_VP, _P4, _VP, _P4, _I, _I, _VP, _VP], _I),
    "kvq_nf4_decode_attn": ([_VP, _P4, _VP, _I, _I, _VP, _VP, _SZ, _VP], _I),
    "kvq_decode_attn_noalloc": ([_VP, _P4, _VP, _VP, _PC, _I, _VP, _VP], _I),
    "kvq_decode_noalloc_scratch_bytes": ([], _SZ),
    "kvq_decode_noalloc_status": ([_VP, ctypes.POINTER(_I)], _I),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libkvq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m packed_cache_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != KVQ_OK:
        raise KvqError(fn, status)


# ----------------------------------------------------------------------------- host queries

def kvq_abi_version() -> int:
    return lib().kvq_abi_version()


def kvq_status_string(status: int) -> str:
    return lib().kvq_status_string(status).decode()


def kvq_codebook(width: int):
    """(centroids as np.float16[2^w], thresholds np.float32[2^w-1], delta float)."""
    n = 1 << width
    c = np.zeros(n, dtype=np.uint16)
    t = np.zeros(n - 1, dtype=np.float32)
    d = np.zeros(1, dtype=np.float32)
    _check("kvq_codebook", lib().kvq_codebook(width, c.ctypes.data, t.ctypes.data, d.ctypes.data))
    return c.view(np.float16), t, float(d[0])


def kvq_nf4_table():
    lv = np.zeros(16, dtype=np.float32)
    mid = np.zeros(15, dtype=np.float32)
    _check("kvq_nf4_table", lib().kvq_nf4_table(lv.ctypes.data, mid.ctypes.data))
    return lv, mid


def cache_desc(batch: int, n_kv_heads: int, capacity: int, bits_k: int, bits_v: int, head_dim: int = HEAD_DIM):
    return CacheDesc(batch, n_kv_heads, head_dim, capacity, bits_k, bits_v)


def kvq_alloc_bytes(n_kv_heads: int) -> int:
    return lib().kvq_alloc_bytes(n_kv_heads)


def kvq_calibrate_workspace_bytes(batch: int, n_kv_heads: int, n_calib_tokens: int) -> int:
    return lib().kvq_calibrate_workspace_bytes(batch, n_kv_heads, n_calib_tokens)


def kvq_packed_bytes(cache: CacheDesc) -> int:
    return lib().kvq_packed_bytes(ctypes.byref(cache))


def kvq_packed_header_bytes(n_kv_heads: int) -> int:
    return lib().kvq_packed_header_bytes(n_kv_heads)


def kvq_packed_status(packed, stream=None) -> int:
    """Status word of a packed cache's header (0, or the kvq_status an append recorded)."""
    code = ctypes.c_int(0)
    lib().kvq_packed_status(packed.data_ptr(), _stream(stream), ctypes.byref(code))
    return code.value


def kvq_debug_decode(wait_limit: int = 2000, no_loads: bool = False) -> None:
    """Test hook: bounded-wait limit (tries of about 1 ms) and the no-copy switch of later decodes."""
    _check("kvq_debug_decode", lib().kvq_debug_decode(int(wait_limit), 1 if no_loads else 0))


def kvq_decode_workspace_bytes(cache: CacheDesc, n_q_heads: int) -> int:
    return lib().kvq_decode_workspace_bytes(ctypes.byref(cache), n_q_heads)


def kvq_nf4_packed_bytes(batch: int, n_heads: int, capacity: int, head_dim: int = HEAD_DIM) -> int:
    return lib().kvq_nf4_packed_bytes(batch, n_heads, capacity, head_dim)


def kvq_nf4_decode_workspace_bytes(batch: int, n_heads: int, capacity: int, head_dim: int = HEAD_DIM) -> int:
    return lib().kvq_nf4_decode_workspace_bytes(batch, n_heads, capacity, head_dim)


def parse_alloc(raw: np.ndarray) -> list[dict]:
    """Decode a host copy of the allocation buffer into per-head dicts of numpy arrays."""
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    size = ctypes.sizeof(HeadAlloc)
    heads = []
    for i in range(len(raw) // size):
        rec = HeadAlloc.from_buffer_copy(raw[i * size:(i + 1) * size].tobytes())
        heads.append({
            "E": np.array(rec.energy[:], dtype=np.float64),
            "g": np.array(rec.gain[:], dtype=np.float32),
            "f": np.array(rec.dequant[:], dtype=np.float32),
            "w": np.array(rec.width[:], dtype=np.int64),
            "bit_off": np.array(rec.bit_off[:], dtype=np.int64),
            "stream_block": np.array(rec.stream_block[:], dtype=np.int64),
            "class_bit": np.array(rec.class_bit[:], dtype=np.int64),
            "class_width": np.array(rec.class_width[:], dtype=np.int64),
            "class_first": np.array(rec.class_first[:], dtype=np.int64),
            "class_blocks": np.array(rec.class_blocks[:], dtype=np.int64),
            "n_classes": rec.n_classes, "n_blocks": rec.n_blocks, "k_words": rec.k_words,
            "plan_col_block": np.array(rec.plan_col_block[:], dtype=np.int64), "plan_k_cols": rec.plan_k_cols,
            "plan_slot": np.array(rec.plan_slot[:], dtype=np.int64), "plan_n_slots": rec.plan_n_slots,
            "digest": int(rec.digest),
            "bits_k": rec.bits_k, "w_max": rec.w_max,
            "mode": rec.mode,
        })
    return heads


# ----------------------------------------------------------------------------- device calls

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    return {torch.float32: KVQ_F32, torch.float16: KVQ_F16, torch.bfloat16: KVQ_BF16}[t.dtype]


def tensor4(t) -> Tensor4:
    """View of a [B][H][T][d] tensor (or [B][H][d], read as T = 1)."""
    if t.dim() == 3:
        B, H, d = t.shape
        return Tensor4(B, H, 1, d, t.stride(0), t.stride(1), d, _dtype_code(t), 0)
    B, H, T, d = t.shape
    if t.stride(3) != 1:
        raise ValueError("last dimension must be contiguous")
    return Tensor4(B, H, T, d, t.stride(0), t.stride(1), t.stride(2), _dtype_code(t), 0)


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _empty_bytes(n: int, device):
    torch = _torch()
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


def kvq_workspace_init(ws, stream=None) -> None:
    _check("kvq_workspace_init", lib().kvq_workspace_init(ws.data_ptr(), ws.numel(), _stream(stream)))


def kvq_workspace_status(ws, stream=None) -> int:
    code = ctypes.c_int(0)
    lib().kvq_workspace_status(ws.data_ptr(), _stream(stream), ctypes.byref(code))
    return code.value


def kvq_calibrate(K, bits_k: int, w_max: int = 8, n_calib: int = 0, mode: int = MODE_BLOCKGTQ,
                  alloc=None, ws=None, stream=None):
    """Calibrate on K [B][Hkv][T][128]; returns the allocation buffer (uint8 device tensor)."""
    B, H, T, _ = K.shape
    n = T if n_calib == 0 else n_calib
    if alloc is None:
        alloc = _empty_bytes(kvq_alloc_bytes(H), K.device)
    if ws is None:
        ws = _torch().zeros(kvq_calibrate_workspace_bytes(B, H, n), dtype=_torch().uint8, device=K.device)
    kd = tensor4(K)
    p = CalibParams(bits_k, w_max, n_calib, mode)
    _check("kvq_calibrate", lib().kvq_calibrate(K.data_ptr(), ctypes.byref(kd), ctypes.byref(p), alloc.data_ptr(),
                                                ws.data_ptr(), ws.numel(), _stream(stream)))
    return alloc


def _opt_tensor(t):
    """(pointer, tensor4 pointer) of an optional tensor; (None, None) for a keys-only call."""
    if t is None:
        return None, None
    return t.data_ptr(), ctypes.byref(tensor4(t))


def kvq_quantize(K, V, alloc, cache: CacheDesc, packed=None, stream=None):
    """Quantize + pack K, V [B][Hkv][T][128] into a packed cache (uint8 device tensor).
    V may be None for a keys-only cache (cache.bits_v = 0)."""
    if packed is None:
        packed = _empty_bytes(kvq_packed_bytes(cache), K.device)
    kd = tensor4(K)
    vp, vd = _opt_tensor(V)
    _check("kvq_quantize", lib().kvq_quantize(K.data_ptr(), ctypes.byref(kd), vp, vd, alloc.data_ptr(),
                                              ctypes.byref(cache), packed.data_ptr(), _stream(stream)))
    return packed


def kvq_append(K, V, alloc, cache: CacheDesc, t_begin: int, packed, stream=None):
    """Quantize K, V [B][Hkv][n][128] as tokens t_begin .. t_begin + n - 1 of `packed`."""
    kd = tensor4(K)
    vp, vd = _opt_tensor(V)
    _check("kvq_append", lib().kvq_append(K.data_ptr(), ctypes.byref(kd), vp, vd, alloc.data_ptr(),
                                          ctypes.byref(cache), int(t_begin), packed.data_ptr(), _stream(stream)))
    return packed


def kvq_decode_attn(q, packed, alloc, cache: CacheDesc, seq_len: int, out=None, ws=None, stream=None):
    """Decode attention for q [B][Hq][128]; returns out fp32 [B][Hq][128]."""
    torch = _torch()
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.zeros(kvq_decode_workspace_bytes(cache, Hq), dtype=torch.uint8, device=q.device)
    qd = tensor4(q)
    _check("kvq_decode_attn", lib().kvq_decode_attn(q.data_ptr(), ctypes.byref(qd), packed.data_ptr(),
                                                    alloc.data_ptr(), ctypes.byref(cache), seq_len, out.data_ptr(),
                                                    ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


def kvq_decode_attn_ex(q, packed, alloc, cache: CacheDesc, seq_len: int, V=None, K_recent=None, V_recent=None,
                       out=None, ws=None, stream=None):
    """Decode attention with the values of a keys-only cache (V [B][Hkv][>= seq_len][128]) and/or
    the most recent tokens kept unquantized (K_recent, V_recent [B][Hkv][R][128])."""
    torch = _torch()
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.zeros(kvq_decode_workspace_bytes(cache, Hq), dtype=torch.uint8, device=q.device)
    ex = DecodeExtra()
    if V is not None:
        ex.V, ex.vd = V.data_ptr(), tensor4(V)
    if K_recent is not None:
        ex.K_recent, ex.krd = K_recent.data_ptr(), tensor4(K_recent)
        ex.V_recent, ex.vrd = V_recent.data_ptr(), tensor4(V_recent)
    qd = tensor4(q)
    _check("kvq_decode_attn_ex", lib().kvq_decode_attn_ex(q.data_ptr(), ctypes.byref(qd), packed.data_ptr(),
                                                          alloc.data_ptr(), ctypes.byref(cache), int(seq_len),
                                                          ctypes.byref(ex), out.data_ptr(), ws.data_ptr(), ws.numel(),
                                                          _stream(stream)))
    return out


def kvq_decode_attn_noalloc(q, packed, alloc, cache: CacheDesc, seq_len: int, out=None, stream=None):
    """Decode attention without a caller workspace: the library's fixed device scratch array
    serves as the split-merge workspace (calls on one device must not overlap)."""
    torch = _torch()
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    qd = tensor4(q)
    _check("kvq_decode_attn_noalloc", lib().kvq_decode_attn_noalloc(q.data_ptr(), ctypes.byref(qd), packed.data_ptr(),
                                                                    alloc.data_ptr(), ctypes.byref(cache), seq_len,
                                                                    out.data_ptr(), _stream(stream)))
    return out


def kvq_decode_noalloc_scratch_bytes() -> int:
    return lib().kvq_decode_noalloc_scratch_bytes()


def kvq_decode_noalloc_status(stream=None) -> int:
    """Status word of the allocation-free decode on the current device (read, then cleared)."""
    code = ctypes.c_int(0)
    lib().kvq_decode_noalloc_status(_stream(stream), ctypes.byref(code))
    return code.value


def kvq_nf4_quantize(K, V, capacity: int | None = None, packed=None, stream=None):
    B, H, T, d = K.shape
    cap = T if capacity is None else capacity
    if packed is None:
        packed = _empty_bytes(kvq_nf4_packed_bytes(B, H, cap, d), K.device)
    kd, vd = tensor4(K), tensor4(V)
    _check("kvq_nf4_quantize", lib().kvq_nf4_quantize(K.data_ptr(), ctypes.byref(kd), V.data_ptr(),
                                                      ctypes.byref(vd), cap, packed.data_ptr(), _stream(stream)))
    return packed


def kvq_nf4_append(K, V, capacity: int, t_begin: int, packed, stream=None):
    """NF4-quantize K, V [B][H][n][128] as tokens t_begin .. t_begin + n - 1 of `packed`."""
    kd, vd = tensor4(K), tensor4(V)
    _check("kvq_nf4_append", lib().kvq_nf4_append(K.data_ptr(), ctypes.byref(kd), V.data_ptr(), ctypes.byref(vd),
                                                  int(capacity), int(t_begin), packed.data_ptr(), _stream(stream)))
    return packed


def kvq_nf4_decode_attn(q, packed, capacity: int, seq_len: int, out=None, ws=None, stream=None):
    torch = _torch()
    B, H, d = q.shape
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.zeros(kvq_nf4_decode_workspace_bytes(B, H, capacity, d), dtype=torch.uint8, device=q.device)
    qd = tensor4(q)
    _check("kvq_nf4_decode_attn", lib().kvq_nf4_decode_attn(q.data_ptr(), ctypes.byref(qd), packed.data_ptr(),
                                                            capacity, seq_len, out.data_ptr(), ws.data_ptr(),
                                                            ws.numel(), _stream(stream)))
    return out


def nf4_sections(packed_np: np.ndarray, batch: int, n_heads: int, capacity: int):
    """Split a host copy of an NF4 buffer into (kcodes, vcodes, kscales, vscales) numpy views."""
    nblk = n_heads * HEAD_DIM // 256
    tp = -(-capacity // 16) * 16
    cb = batch * nblk * tp * 128
    kc = packed_np[:cb].reshape(batch, nblk, tp, 128)
    vc = packed_np[cb:2 * cb].reshape(batch, nblk, tp, 128)
    sc = packed_np[2 * cb:2 * cb + 4 * batch * nblk * tp].view("<f2")
    ks = sc[:batch * nblk * tp].reshape(batch, nblk, tp)
    vs = sc[batch * nblk * tp:].reshape(batch, nblk, tp)
    return kc, vc, ks, vs
