"""Python binding of libzz: zigzag context-parallel prefill attention on B200.

Argument marshalling only.  Every step of the path runs in the CUDA kernels
of ``libzz.so`` (built in-tree by ``zigzag_context_causal_b200.build``);
PyTorch supplies device memory and streams.  There is no fallback: if the
shared library is missing, importing this package raises.

Typical use on one GPU (all ``c`` virtual ranks in one launch)::

    plan = Plan(cp_size=8, extend_lens=[131072])
    ws = plan.upload()                                   # device tables
    shard_rows(plan, q_tokens, q_ranked)                 # [T,Hq,D] -> [c*M,Hq,D]
    rerange_kv_to_pool(plan, k_gath, v_gath, k_pool, v_pool, out_cache_loc)
    attn_prefill(plan, q_ranked, k_pool, v_pool, page_table, page_size, out)
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzz.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "zz.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libzz.so not found at {LIB_PATH}; build it with "
        "`python -m zigzag_context_causal_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

ZZ_OK, ZZ_ERR_INVALID_ARG, ZZ_ERR_NOT_APPLICABLE, ZZ_ERR_UNSUPPORTED, ZZ_ERR_CUDA, \
    ZZ_ERR_DEVICE_TIMEOUT = range(6)
ZZ_BF16, ZZ_FP32 = 0, 1
FIELDS = {
    "extend_lens": 0, "prefix": 1, "split_list": 2, "zigzag_index": 3, "cp_reverse_index": 4,
    "reverse_split_len": 5, "per_rank_actual_token": 6, "max_rank_len": 7, "kv_len_prev": 8,
    "kv_len_next": 9, "q_len_prev": 10, "q_len_next": 11, "cu_seqlens_q_prev": 12,
    "cu_seqlens_q_next": 13, "src_row": 14, "rank_tok": 15,
}
PER_RANK_FIELDS = {"zigzag_index", "kv_len_prev", "kv_len_next", "q_len_prev", "q_len_next",
                   "cu_seqlens_q_prev", "cu_seqlens_q_next"}


class ZZError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[zz status {status}] {msg}")
        self.status = status


class _Info(ctypes.Structure):
    _fields_ = [("cp_size", ctypes.c_int32), ("bs", ctypes.c_int32),
                ("total_tokens", ctypes.c_int64), ("max_rank_len", ctypes.c_int32),
                ("total_q_prev", ctypes.c_int32), ("total_q_next", ctypes.c_int32),
                ("max_seqlen_q_prev", ctypes.c_int32), ("max_seqlen_q_next", ctypes.c_int32),
                ("causal_pairs", ctypes.c_int64)]


_P = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)
_sig = {
    "zz_last_error": (ctypes.c_char_p, []),
    "zz_plan_create": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _I32P, _I32P, ctypes.c_int64,
                                      ctypes.POINTER(_P)]),
    "zz_plan_destroy": (None, [_P]),
    "zz_plan_info": (ctypes.c_int, [_P, ctypes.c_int, ctypes.POINTER(_Info)]),
    "zz_plan_get": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, _I32P, ctypes.c_int64,
                                   ctypes.POINTER(ctypes.c_int64)]),
    "zz_plan_workspace_bytes": (ctypes.c_size_t, [_P]),
    "zz_plan_upload": (ctypes.c_int, [_P, _P, ctypes.c_size_t, _P]),
    "zz_plan_device_status": (ctypes.c_int, [_P, _I32P, ctypes.c_int, _P]),
    "zz_shard_rows": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P]),
    "zz_gather_rows": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P]),
    "zz_take_back_rows": (ctypes.c_int, [_P, ctypes.c_int, _P, _P, ctypes.c_int64, _P]),
    "zz_rerange_kv_to_pool": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int64, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, _P]),
    "zz_rerange_kv_to_pool_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int64, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_float, ctypes.c_float, _P]),
    "zz_attn_prefill": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, ctypes.c_int64,
                                       _P, ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int, _P]),
}
_sig["zz_attn_prefill_noalloc"] = _sig["zz_attn_prefill"]
_sig["zz_attn_prefill_ex"] = (ctypes.c_int, _sig["zz_attn_prefill"][1][:-1] + [ctypes.c_uint32, _P])
_sig["zz_debug_wait_timeout"] = (ctypes.c_int, [ctypes.c_int64, _P, _P])
_PP = ctypes.POINTER(_P)
_sig["zz_rerange_push_kv"] = (ctypes.c_int, [_P, ctypes.c_int, _P, _P, _PP, _PP, _PP, ctypes.c_int,
                                             ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P])
_sig["zz_ipc_export"] = (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int64)])
_sig["zz_ipc_import"] = (ctypes.c_int, [_P, ctypes.c_int64, _PP, _PP])
_sig["zz_ipc_close"] = (ctypes.c_int, [_P])
ZZ_MAX_PUSH_DST = 16
ZZ_IPC_HANDLE_BYTES = 64
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_functions() -> list[str]:
    """Names of the functions ``include/zz.h`` declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:zz_status_t|void|size_t|const char\*)\s+(zz_\w+)\s*\(",
                                 text, flags=re.M)))


def _check(st: int) -> None:
    if st != ZZ_OK:
        raise ZZError(st, _lib.zz_last_error().decode())


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return getattr(stream, "cuda_stream", stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libzz must be contiguous")
    return t.data_ptr()


def _i32_array(xs):
    if xs is None:
        return None
    arr = (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])
    return ctypes.cast(arr, _I32P)


_DT = {torch.bfloat16: ZZ_BF16, torch.float32: ZZ_FP32}


class Plan:
    """Host-side zigzag plan for all ``cp_size`` ranks (zz_plan_create)."""

    def __init__(self, cp_size: int, extend_lens=None, seq_lens=None, num_tokens: int | None = None):
        if extend_lens is None and seq_lens is None and num_tokens is None:
            raise ValueError("give extend_lens, seq_lens or num_tokens")
        lens = extend_lens if extend_lens is not None else seq_lens
        bs = len(lens) if lens is not None else 1
        if num_tokens is None:
            num_tokens = sum(int(x) for x in lens)
        handle = _P()
        self._keep = (_i32_array(extend_lens), _i32_array(seq_lens))
        _check(_lib.zz_plan_create(int(cp_size), bs, self._keep[0], self._keep[1],
                                   int(num_tokens), ctypes.byref(handle)))
        self._h = handle
        self.workspace = None
        info = self.info(0)
        self.cp_size, self.bs = info.cp_size, info.bs
        self.total_tokens, self.M = info.total_tokens, info.max_rank_len
        self.causal_pairs = info.causal_pairs

    def __del__(self, _destroy=_lib.zz_plan_destroy):
        h = getattr(self, "_h", None)
        if h:
            _destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def info(self, rank: int = 0) -> _Info:
        out = _Info()
        _check(_lib.zz_plan_info(self._h, rank, ctypes.byref(out)))
        return out

    def get(self, field: str, rank: int = 0) -> list[int]:
        n = ctypes.c_int64()
        fid = FIELDS[field]
        _check(_lib.zz_plan_get(self._h, rank, fid, None, 0, ctypes.byref(n)))
        buf = (ctypes.c_int32 * max(n.value, 1))()
        _check(_lib.zz_plan_get(self._h, rank, fid, ctypes.cast(buf, _I32P), n.value, ctypes.byref(n)))
        return list(buf[: n.value])

    def get_all_ranks(self, field: str) -> list[list[int]]:
        return [self.get(field, r) for r in range(self.cp_size)]

    def workspace_bytes(self) -> int:
        return int(_lib.zz_plan_workspace_bytes(self._h))

    def upload(self, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Copy the device tables into ``workspace`` (allocated here if None)."""
        nbytes = self.workspace_bytes()
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        _check(_lib.zz_plan_upload(self._h, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)))
        self.workspace = workspace
        return workspace

    def device_status(self, clear: bool = True, stream=None) -> int:
        flags = ctypes.c_int32()
        st = _lib.zz_plan_device_status(self._h, ctypes.byref(flags), int(clear), _stream(stream))
        if st not in (ZZ_OK, ZZ_ERR_DEVICE_TIMEOUT):
            _check(st)
        return flags.value


def shard_rows(plan: Plan, src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    """``dst[src_row[t]] = src[t]``: natural order -> rank-ordered padded rows."""
    row_bytes = src[0].numel() * src.element_size()
    _check(_lib.zz_shard_rows(plan.handle, _ptr(src), _ptr(dst), row_bytes, _stream(stream)))


def gather_rows(plan: Plan, src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    """``dst[t] = src[src_row[t]]``: rank-ordered padded rows -> natural order."""
    row_bytes = src[0].numel() * src.element_size()
    _check(_lib.zz_gather_rows(plan.handle, _ptr(src), _ptr(dst), row_bytes, _stream(stream)))


def take_back_rows(plan: Plan, rank: int, src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    """Rank ``rank``'s rank-local rows out of a natural-order tensor."""
    row_bytes = src[0].numel() * src.element_size()
    _check(_lib.zz_take_back_rows(plan.handle, int(rank), _ptr(src), _ptr(dst), row_bytes,
                                  _stream(stream)))


def rerange_kv_to_pool(plan: Plan, k_gathered, v_gathered, k_pool, v_pool, out_cache_loc,
                       stream=None) -> None:
    """Fused trim + rerange + pool write of the all-gathered K (and V)."""
    h_kv, d = k_gathered.shape[-2], k_gathered.shape[-1]
    _check(_lib.zz_rerange_kv_to_pool(plan.handle, _ptr(k_gathered), _ptr(v_gathered), _ptr(k_pool),
                                      _ptr(v_pool), _ptr(out_cache_loc), k_pool.shape[0], h_kv, d,
                                      _DT[k_gathered.dtype], _stream(stream)))


def rerange_kv_to_pool_fp8(plan: Plan, k_gathered, v_gathered, k_pool, v_pool, out_cache_loc,
                           k_scale: float, v_scale: float = 1.0, stream=None) -> None:
    """Fused rerange of bf16 K (and V) into E4M3 pools: ``e4m3(x / scale)``."""
    h_kv, d = k_gathered.shape[-2], k_gathered.shape[-1]
    _check(_lib.zz_rerange_kv_to_pool_fp8(plan.handle, _ptr(k_gathered), _ptr(v_gathered), _ptr(k_pool),
                                          _ptr(v_pool), _ptr(out_cache_loc), k_pool.shape[0], h_kv, d,
                                          float(k_scale), float(v_scale), _stream(stream)))


def _addr(x) -> int:
    """Device address of a tensor, or an int already holding one (a mapped peer buffer)."""
    return x if isinstance(x, int) else _ptr(x)


def rerange_push_kv(plan: Plan, rank: int, k_local, v_local, k_pools, v_pools, out_cache_locs,
                    num_slots: int, stream=None) -> None:
    """Rank ``rank`` writes its local K (and V) rows into every pool of the lists.

    ``k_local``/``v_local``: ``[>= per_rank_actual_token[rank], H_kv, D]``;
    ``k_pools``/``v_pools``/``out_cache_locs``: one entry per destination, each a
    tensor on this GPU or an int address (a peer pool mapped with ``PeerBuffer``).
    """
    n = len(k_pools)
    if (v_pools is not None and len(v_pools) != n) or len(out_cache_locs) != n:
        raise ValueError("k_pools, v_pools and out_cache_locs must have one entry per destination")
    kp = (_P * n)(*[_addr(x) for x in k_pools])
    vp = (_P * n)(*[_addr(x) for x in v_pools]) if v_pools is not None else None
    lp = (_P * n)(*[_addr(x) for x in out_cache_locs])
    h_kv, d = k_local.shape[-2], k_local.shape[-1]
    _check(_lib.zz_rerange_push_kv(plan.handle, int(rank), _ptr(k_local), _ptr(v_local), kp, vp, lp, n,
                                   int(num_slots), h_kv, d, _DT[k_local.dtype], _stream(stream)))


def ipc_export(t: torch.Tensor) -> tuple[bytes, int]:
    """(handle, offset) naming ``t``'s device memory for another process."""
    buf = ctypes.create_string_buffer(ZZ_IPC_HANDLE_BYTES)
    off = ctypes.c_int64(0)
    _check(_lib.zz_ipc_export(_ptr(t), buf, ctypes.byref(off)))
    return buf.raw, off.value


class PeerBuffer:
    """Another process's exported buffer mapped into this one; ``ptr`` is its address."""

    def __init__(self, handle: bytes, offset: int):
        if len(handle) != ZZ_IPC_HANDLE_BYTES:
            raise ValueError("IPC handle must be 64 bytes")
        base, ptr = _P(), _P()
        _check(_lib.zz_ipc_import(handle, int(offset), ctypes.byref(base), ctypes.byref(ptr)))
        self._base = base.value
        self.ptr = ptr.value

    def close(self) -> None:
        if self._base:
            _check(_lib.zz_ipc_close(self._base))
            self._base = None


ZZ_ATTN_NONCAUSAL = 1


def attn_prefill(plan: Plan, q, k_pool, v_pool, page_table, page_size: int, out, lse=None,
                 softmax_scale: float = 0.0, rank_begin: int = 0, rank_count: int | None = None,
                 stream=None, causal: bool = True) -> None:
    """Both zigzag halves of ranks [rank_begin, rank_begin+rank_count) in one launch.

    ``q``/``out``: ``[rank_count*M, H_q, D]`` (or ``[rank_count, M, H_q, D]``),
    ``k_pool``/``v_pool``: ``[slots, H_kv, D]``, ``page_table``: ``[bs, max_pages]`` int32.
    """
    if rank_count is None:
        rank_count = plan.cp_size
    h_q, d = q.shape[-2], q.shape[-1]
    h_kv = k_pool.shape[-2]
    _check(_lib.zz_attn_prefill_ex(plan.handle, rank_begin, rank_count, _ptr(q), _ptr(k_pool),
                                   _ptr(v_pool), k_pool.shape[0], _ptr(page_table), page_table.shape[1],
                                   int(page_size), _ptr(out), _ptr(lse), h_q, h_kv, d,
                                   float(softmax_scale), _DT[q.dtype], 0 if causal else ZZ_ATTN_NONCAUSAL,
                                   _stream(stream)))


def raw_call(name: str, *args) -> int:
    """Call a C-ABI entry point by name with raw ctypes arguments (tests)."""
    return getattr(_lib, name)(*args)


def last_error() -> str:
    return _lib.zz_last_error().decode()


def debug_wait_timeout(timeout_ns: int, status: torch.Tensor, stream=None) -> None:
    """Run the bounded-wait self test; ``status`` is an int64 CUDA tensor of 2."""
    _check(_lib.zz_debug_wait_timeout(int(timeout_ns), _ptr(status), _stream(stream)))
