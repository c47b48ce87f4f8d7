"""Python binding of libpagedattn (paged decode attention, B200 / sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libpagedattn.so``; torch is used for device memory and streams.
If the library has not been built the calls raise -- there is no fallback.

``decode`` takes its arguments in the order of the call printed in the PR
#47361 benchmark snippet (out, query, key_cache, value_cache, num_kv_heads,
scale, block_tables, seq_lens, block_size, max_seq_len, kv dtype, k_scale,
v_scale), with the split-KV temporaries folded into one optional workspace.
"""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_WORKSPACE_TOO_SMALL = 3
PA_ERR_CUDA = 4
PA_ERR_OUT_OF_BLOCKS = 5

PA_KV_BF16 = 0
PA_KV_FP8_E4M3 = 1

PA_DEV_BAD_BLOCK_ID = 0x1
PA_DEV_SEQ_LEN_OUT_OF_RANGE = 0x2
PA_DEV_WAIT_TIMEOUT = 0x4
PA_DEV_PREFIX_MISMATCH = 0x8

WORKSPACE_HEADER_BYTES = 256
WORKSPACE_MERGE_COUNT_BYTES = 4096  # after the header when the plan needs more
NOALLOC_SCRATCH_BYTES = 16 << 20

_KV = {"bf16": PA_KV_BF16, "auto": PA_KV_BF16, "fp8": PA_KV_FP8_E4M3, "fp8_e4m3": PA_KV_FP8_E4M3,
       PA_KV_BF16: PA_KV_BF16, PA_KV_FP8_E4M3: PA_KV_FP8_E4M3}


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(detail)


class Options(ctypes.Structure):
    _fields_ = [("partition_pages", ctypes.c_int), ("num_sms", ctypes.c_int),
                ("stages", ctypes.c_int), ("shared_prefix_blocks", ctypes.c_int),
                ("alibi_slopes", ctypes.c_void_p), ("fp8_compute", ctypes.c_int),
                ("test_stall_copies", ctypes.c_int), ("schedule", ctypes.c_int),
                ("mha_cuda_cores", ctypes.c_int)]


class Plan(ctypes.Structure):
    _fields_ = [("num_partitions", ctypes.c_int), ("partition_pages", ctypes.c_int),
                ("stages", ctypes.c_int), ("warps_per_cta", ctypes.c_int),
                ("grid_ctas", ctypes.c_longlong), ("smem_bytes", ctypes.c_size_t),
                ("workspace_bytes", ctypes.c_size_t), ("prefix_partitions", ctypes.c_int),
                ("prefix_groups", ctypes.c_int), ("balanced", ctypes.c_int),
                ("dynamic", ctypes.c_int), ("tail_units", ctypes.c_longlong),
                ("tail_partitions", ctypes.c_int), ("tail_partition_pages", ctypes.c_int),
                ("combine", ctypes.c_int), ("longest_first", ctypes.c_int)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int


def _bind(lib):
    decode_args = [_P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, _P, _I, _P, _I, _I,
                   ctypes.c_int64, _I, _P, _P, _P, ctypes.c_size_t, _P]
    lib.pa_decode.argtypes = decode_args
    lib.pa_decode.restype = _I
    lib.pa_decode_ex.argtypes = decode_args + [ctypes.POINTER(Options)]
    lib.pa_decode_ex.restype = _I
    lib.pa_decode_noalloc.argtypes = decode_args[:18] + [_P]
    lib.pa_decode_noalloc.restype = _I
    lib.pa_plan_decode.argtypes = [ctypes.POINTER(Plan), _I, _I, _I, _I, _I, _I, _I,
                                   ctypes.POINTER(Options)]
    lib.pa_plan_decode.restype = _I
    lib.pa_decode_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(Options)]
    lib.pa_decode_workspace_size.restype = ctypes.c_size_t
    lib.pa_read_device_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32), _I, _P]
    lib.pa_read_device_status.restype = _I
    lib.pa_status_string.argtypes = [_I]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_last_error_detail.argtypes = []
    lib.pa_last_error_detail.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = _I
    I64 = ctypes.c_int64
    lib.pa_bm_create.argtypes = [ctypes.POINTER(_P), I64, _I, _I]
    lib.pa_bm_create.restype = _I
    lib.pa_bm_destroy.argtypes = [_P]
    lib.pa_bm_destroy.restype = None
    lib.pa_bm_add_sequence.argtypes = [_P, ctypes.POINTER(_I)]
    lib.pa_bm_add_sequence.restype = _I
    lib.pa_bm_fork.argtypes = [_P, _I, ctypes.POINTER(_I)]
    lib.pa_bm_fork.restype = _I
    lib.pa_bm_free_sequence.argtypes = [_P, _I]
    lib.pa_bm_free_sequence.restype = _I
    lib.pa_bm_append_tokens.argtypes = [_P, _I, _I, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                        ctypes.POINTER(_I)]
    lib.pa_bm_append_tokens.restype = _I
    lib.pa_bm_seq_len.argtypes = [_P, _I, ctypes.POINTER(I64)]
    lib.pa_bm_seq_len.restype = _I
    lib.pa_bm_export.argtypes = [_P, _P, _I, _P, _I, _P]
    lib.pa_bm_export.restype = _I
    lib.pa_bm_num_free_blocks.argtypes = [_P]
    lib.pa_bm_num_free_blocks.restype = I64
    lib.pa_bm_refcount.argtypes = [_P, I64]
    lib.pa_bm_refcount.restype = _I
    lib.pa_bm_last_error_detail.argtypes = []
    lib.pa_bm_last_error_detail.restype = ctypes.c_char_p
    lib.pa_copy_blocks.argtypes = [_P, _P, _I, _I, _I, I64, _I, _P, _P, _I, _P, _P]
    lib.pa_copy_blocks.restype = _I
    return lib


def lib():
    """The loaded libpagedattn (raises if it was never built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m paged_kv_cache_471_b200.build` (there is no fallback path)")
                _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def _check(rc: int):
    if rc != PA_OK:
        L = lib()
        raise PagedAttentionError(rc, f"{L.pa_status_string(rc).decode()}: "
                                      f"{L.pa_last_error_detail().decode()}")


SCHEDULES = {"auto": 0, "balanced": 1, "partitioned": 2, "dynamic": 3}


def _opts(partition_pages=0, num_sms=0, stages=0, shared_prefix_blocks=0, alibi_ptr=None,
          fp8_compute=False, test_stall_copies=False, schedule="auto", mha_cuda_cores=False):
    if schedule not in SCHEDULES:
        raise ValueError(f"schedule must be one of {sorted(SCHEDULES)}")
    if not partition_pages and not num_sms and not stages and not shared_prefix_blocks \
            and not alibi_ptr and not fp8_compute and not test_stall_copies \
            and schedule == "auto" and not mha_cuda_cores:
        return None
    return ctypes.byref(Options(int(partition_pages), int(num_sms), int(stages),
                                int(shared_prefix_blocks), alibi_ptr, int(bool(fp8_compute)),
                                int(bool(test_stall_copies)), SCHEDULES[schedule],
                                int(bool(mha_cuda_cores))))


def kv_dtype_code(kv_dtype) -> int:
    try:
        return _KV[kv_dtype]
    except KeyError:
        raise ValueError(f"unsupported kv dtype {kv_dtype!r}") from None


def plan(num_seqs, num_heads, num_kv_heads, head_size, block_size, max_seq_len, kv_dtype="bf16",
         partition_pages=0, num_sms=0, stages=0, shared_prefix_blocks=0, fp8_compute=False,
         schedule="auto") -> dict:
    p = Plan()
    _check(lib().pa_plan_decode(ctypes.byref(p), num_seqs, num_heads, num_kv_heads, head_size,
                                block_size, max_seq_len, kv_dtype_code(kv_dtype),
                                _opts(partition_pages, num_sms, stages, shared_prefix_blocks,
                                      None, fp8_compute, False, schedule)))
    return p.as_dict()


def workspace_size(num_seqs, num_heads, num_kv_heads, head_size, block_size, max_seq_len,
                   kv_dtype="bf16", partition_pages=0, num_sms=0, shared_prefix_blocks=0,
                   fp8_compute=False, schedule="auto", stages=0) -> int:
    n = lib().pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_size, block_size,
                                       max_seq_len, kv_dtype_code(kv_dtype),
                                       _opts(partition_pages, num_sms, stages, shared_prefix_blocks,
                                             None, fp8_compute, False, schedule))
    if n == 0:
        raise PagedAttentionError(PA_ERR_INVALID_ARG, lib().pa_last_error_detail().decode())
    return n


_ws_cache = {}


def workspace(nbytes: int, device):
    """A zeroed workspace of at least nbytes on `device`, reused across calls
    (its status word is sticky; see read_status)."""
    import torch
    dev = torch.device(device)
    key = (dev.type, dev.index)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, WORKSPACE_HEADER_BYTES), dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def _ptr(t, name, dtypes=None, device=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return t.data_ptr()


def decode(out, query, key_cache, value_cache, num_kv_heads: int, scale: float, block_tables,
           seq_lens, block_size: int, max_seq_len: int, kv_dtype="bf16", k_scale=None,
           v_scale=None, workspace_tensor=None, partition_pages: int = 0, stream=None,
           stages: int = 0, shared_prefix_blocks: int = 0, alibi_slopes=None,
           fp8_compute: bool = False, test_stall_copies: bool = False, schedule: str = "auto",
           mha_cuda_cores: bool = False, num_sms: int = 0):
    """Paged decode attention into ``out`` (bf16 [num_seqs, num_heads, head_size]).

    key_cache: [num_blocks, num_kv_heads, head_size/x, block_size, x];
    value_cache: [num_blocks, num_kv_heads, head_size, block_size]; bf16, or
    uint8 / float8_e4m3fn holding e4m3 codes when kv_dtype is "fp8_e4m3"
    (then k_scale / v_scale are 1-element fp32 CUDA tensors).

    The keyword options are those of pa_options in include/pagedattn.h:
    partition_pages, stages, shared_prefix_blocks, alibi_slopes ([num_heads]
    fp32), fp8_compute, test_stall_copies, schedule ("auto",
    "partitioned", "balanced" or "dynamic"), mha_cuda_cores and num_sms (plan
    as if the GPU had that many SMs; 0 = the device's count).  workspace_tensor
    defaults to a cached zeroed buffer per device; stream defaults to the
    current stream.
    """
    import torch
    code = kv_dtype_code(kv_dtype)
    dev = query.device
    S, Hq, D = query.shape
    kv_types = (torch.bfloat16,) if code == PA_KV_BF16 else (torch.uint8, torch.float8_e4m3fn)
    args_ptrs = [
        _ptr(out, "out", (torch.bfloat16,), dev),
        _ptr(query, "query", (torch.bfloat16,), dev),
        _ptr(key_cache, "key_cache", kv_types, dev),
        _ptr(value_cache, "value_cache", kv_types, dev),
    ]
    if tuple(out.shape) != (S, Hq, D):
        raise ValueError("out must have the query's shape")
    if key_cache.dim() != 5 or value_cache.dim() != 4:
        raise ValueError("key_cache must be 5-D and value_cache 4-D")
    num_blocks = key_cache.shape[0]
    if value_cache.shape[0] != num_blocks or key_cache.shape[3] != block_size \
            or value_cache.shape[3] != block_size or key_cache.shape[1] != num_kv_heads \
            or value_cache.shape[1] != num_kv_heads or value_cache.shape[2] != D \
            or key_cache.shape[2] * key_cache.shape[4] != D:
        raise ValueError("cache shapes do not match query / num_kv_heads / block_size")
    bt = _ptr(block_tables, "block_tables", (torch.int32,), dev)
    sl = _ptr(seq_lens, "seq_lens", (torch.int32,), dev)
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks] and seq_lens [num_seqs]")
    ks = vs = None
    if code == PA_KV_FP8_E4M3:
        ks = _ptr(k_scale, "k_scale", (torch.float32,), dev)
        vs = _ptr(v_scale, "v_scale", (torch.float32,), dev)
    alibi = None
    if alibi_slopes is not None:
        if alibi_slopes.shape != (Hq,):
            raise ValueError("alibi_slopes must be [num_heads]")
        alibi = _ptr(alibi_slopes, "alibi_slopes", (torch.float32,), dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    # The library plans for, and launches on, the current device: make it the
    # tensors' device for the call.
    with torch.cuda.device(dev):
        if workspace_tensor is None:  # (a given one is size-checked by the library)
            need = workspace_size(S, Hq, num_kv_heads, D, block_size, max_seq_len, code,
                                  partition_pages, shared_prefix_blocks=shared_prefix_blocks,
                                  fp8_compute=fp8_compute and code == PA_KV_FP8_E4M3,
                                  schedule=schedule, stages=stages, num_sms=num_sms)
            workspace_tensor = workspace(need, dev)
        ws = _ptr(workspace_tensor, "workspace", None, dev)
        rc = lib().pa_decode_ex(*args_ptrs, S, Hq, int(num_kv_heads), D, float(scale), bt,
                                block_tables.shape[1], sl, int(block_size), int(max_seq_len),
                                int(num_blocks), code, ks, vs, ws,
                                workspace_tensor.numel() * workspace_tensor.element_size(),
                                st.cuda_stream,
                                _opts(partition_pages, num_sms, stages, shared_prefix_blocks, alibi,
                                      fp8_compute, test_stall_copies, schedule, mha_cuda_cores))
    _check(rc)
    return out


def decode_noalloc(out, query, key_cache, value_cache, num_kv_heads: int, scale: float,
                   block_tables, seq_lens, block_size: int, max_seq_len: int, kv_dtype="bf16",
                   k_scale=None, v_scale=None, stream=None):
    """``decode`` for callers that may not allocate device memory when they
    call: the split-KV scratch is the library's own fixed device array
    (NOALLOC_SCRATCH_BYTES per GPU), so nothing is allocated here.  Calls that
    overlap on the GPU share that array and must be serialised by the caller;
    the first call on a device should come before any stream capture."""
    import torch
    code = kv_dtype_code(kv_dtype)
    dev = query.device
    S, Hq, D = query.shape
    kv_types = (torch.bfloat16,) if code == PA_KV_BF16 else (torch.uint8, torch.float8_e4m3fn)
    ks = vs = None
    if code == PA_KV_FP8_E4M3:
        ks = _ptr(k_scale, "k_scale", (torch.float32,), dev)
        vs = _ptr(v_scale, "v_scale", (torch.float32,), dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    ptrs = (_ptr(out, "out", (torch.bfloat16,), dev), _ptr(query, "query", (torch.bfloat16,), dev),
            _ptr(key_cache, "key_cache", kv_types, dev),
            _ptr(value_cache, "value_cache", kv_types, dev))
    bt = _ptr(block_tables, "block_tables", (torch.int32,), dev)
    sl = _ptr(seq_lens, "seq_lens", (torch.int32,), dev)
    with torch.cuda.device(dev):  # the scratch array of the tensors' device
        rc = lib().pa_decode_noalloc(*ptrs, S, Hq, int(num_kv_heads), D, float(scale), bt,
                                     block_tables.shape[1], sl, int(block_size), int(max_seq_len),
                                     int(key_cache.shape[0]), code, ks, vs, st.cuda_stream)
    _check(rc)
    return out


def read_status(workspace_tensor=None, device=None, clear=False, stream=None) -> int:
    """The sticky PA_DEV_* bits kernels set in a workspace (synchronises)."""
    import torch
    if workspace_tensor is None:
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        workspace_tensor = workspace(WORKSPACE_HEADER_BYTES, dev)
    st = stream if stream is not None else torch.cuda.current_stream(workspace_tensor.device)
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(workspace_tensor.device):
        rc = lib().pa_read_device_status(ctypes.c_void_p(workspace_tensor.data_ptr()),
                                         ctypes.byref(flags), int(bool(clear)), st.cuda_stream)
    _check(rc)
    return int(flags.value)


def version() -> int:
    return int(lib().pa_version())


# --------------------------------------------------------------- block manager
def _bm_check(rc: int):
    if rc != PA_OK:
        L = lib()
        raise PagedAttentionError(rc, f"{L.pa_status_string(rc).decode()}: "
                                      f"{L.pa_bm_last_error_detail().decode()}")


class BlockManager:
    """Host block allocator of libpagedattn (``pa_bm_*``): blocks on demand,
    forked sequences sharing blocks, copy on write of a shared partial block."""

    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int):
        self._h = ctypes.c_void_p()
        _bm_check(lib().pa_bm_create(ctypes.byref(self._h), int(num_blocks), int(block_size),
                                     int(max_blocks_per_seq)))
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self.max_blocks_per_seq = int(max_blocks_per_seq)

    def close(self):
        if self._h:
            lib().pa_bm_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_sequence(self) -> int:
        i = ctypes.c_int()
        _bm_check(lib().pa_bm_add_sequence(self._h, ctypes.byref(i)))
        return i.value

    def fork(self, parent: int) -> int:
        i = ctypes.c_int()
        _bm_check(lib().pa_bm_fork(self._h, int(parent), ctypes.byref(i)))
        return i.value

    def free(self, seq: int):
        _bm_check(lib().pa_bm_free_sequence(self._h, int(seq)))

    def append(self, seq: int, num_tokens: int):
        """Grow a sequence; returns (src, dst) when a copy on write is needed."""
        a, b, n = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int()
        _bm_check(lib().pa_bm_append_tokens(self._h, int(seq), int(num_tokens), ctypes.byref(a),
                                            ctypes.byref(b), ctypes.byref(n)))
        return (a.value, b.value) if n.value else None

    def seq_len(self, seq: int) -> int:
        n = ctypes.c_int64()
        _bm_check(lib().pa_bm_seq_len(self._h, int(seq), ctypes.byref(n)))
        return n.value

    def export(self, seqs):
        """(block_tables int32 [n, max_blocks_per_seq], seq_lens int32 [n]) on the host."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        bt = np.empty((len(ids), self.max_blocks_per_seq), dtype=np.int32)
        sl = np.empty((len(ids),), dtype=np.int32)
        _bm_check(lib().pa_bm_export(self._h, ids.ctypes.data, len(ids), bt.ctypes.data,
                                     self.max_blocks_per_seq, sl.ctypes.data))
        return bt, sl

    def num_free_blocks(self) -> int:
        return int(lib().pa_bm_num_free_blocks(self._h))

    def refcount(self, block: int) -> int:
        return int(lib().pa_bm_refcount(self._h, int(block)))


def copy_blocks(key_cache, value_cache, src, dst, kv_dtype="bf16", status=None, stream=None):
    """Copy whole blocks (all kv heads, K and V): block dst[i] <- block src[i].
    src / dst: int64 CUDA tensors of block ids."""
    import torch
    code = kv_dtype_code(kv_dtype)
    dev = key_cache.device
    kv_types = (torch.bfloat16,) if code == PA_KV_BF16 else (torch.uint8, torch.float8_e4m3fn)
    n = int(src.numel())
    if int(dst.numel()) != n:
        raise ValueError("src and dst must have the same length")
    Hk, D = value_cache.shape[1], value_cache.shape[2]
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    args = (_ptr(key_cache, "key_cache", kv_types, dev),
            _ptr(value_cache, "value_cache", kv_types, dev),
            int(Hk), int(D), int(value_cache.shape[3]), int(key_cache.shape[0]), code,
            _ptr(src, "src", (torch.int64,), dev), _ptr(dst, "dst", (torch.int64,), dev), n,
            None if status is None else _ptr(status, "status", None, dev), st.cuda_stream)
    with torch.cuda.device(dev):
        rc = lib().pa_copy_blocks(*args)
    _bm_check(rc)
