"""B200-native paged KV-cache decode attention.

Python binding of the C ABI declared in ``include/pa.h`` (library ``libpa.so`` in this
directory, built by ``python -m paged_kv_cache_427_b200.build``).  The binding only marshals
torch tensors into ``pa_tensor`` descriptors and passes the current CUDA stream: every step of
the computation runs in the library's sm_100a kernels.  There is no CPU fallback: if the
library is missing or fails to load, every call raises.

Calls (same names as the C ABI):
  pa_reshape_and_cache(key, value, key_cache, value_cache, slot_mapping)
  pa_copy_blocks(key_cache, value_cache, block_mapping)
  pa_decode(out, query, key_cache, value_cache, block_tables, context_lens, scale,
            block_size, num_kv_heads)
  pa_decode_ex(..., num_workers=0, flags=0, workspace=None)
  pa_decode_workspace_bytes, pa_decode_default_workers, pa_workspace_init,
  pa_release_workspaces, pa_last_error, pa_get_device_error, pa_version
Measurement aids: pa_set_decode_timeline(buf), pa_hbm_read_probe(buf, mode, sink).
Seeded synthetic workloads live in ``paged_kv_cache_427_b200.workloads`` (no torch, no CUDA).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libpa.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "pa.h")

PA_F32, PA_BF16, PA_F16, PA_I32, PA_I64, PA_FP8_E4M3 = 0, 1, 2, 3, 4, 5
PA_OK = 0
PA_DECODE_SEPARATE_REDUCE = 0x1
PA_DECODE_CUDA_CORES = 0x2
PA_DECODE_OVERLAP_PREVIOUS = 0x4
PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_CONTEXT_LEN = 0x2
PA_DEVERR_SLOT = 0x4
PA_DEVERR_COPY_PAIR = 0x8
PA_DEVERR_TIMEOUT = 0x10
PA_DEVERR_PREFIX = 0x20
PA_NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024
PA_ERR_INVALID_ARG = -1
PA_ERR_SHAPE = -2
PA_ERR_DTYPE = -3
PA_ERR_UNSUPPORTED = -4
PA_ERR_CUDA = -5
PA_ERR_WORKSPACE = -6
PA_ERR_LAYOUT = -7
STATUS_NAMES = {0: "PA_OK", -1: "PA_ERR_INVALID_ARG", -2: "PA_ERR_SHAPE", -3: "PA_ERR_DTYPE",
                -4: "PA_ERR_UNSUPPORTED", -5: "PA_ERR_CUDA", -6: "PA_ERR_WORKSPACE",
                -7: "PA_ERR_LAYOUT"}


class PaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 5), ("stride", ctypes.c_int64 * 5)]


class PagedAttentionError(RuntimeError):
    def __init__(self, call: str, status: int, message: str):
        super().__init__(f"{call} failed: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_T = ctypes.POINTER(PaTensor)


def load(path: str = LIBRARY) -> ctypes.CDLL:
    """Load libpa.so (once).  Raises ImportError when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m paged_kv_cache_427_b200.build`")
    lib = ctypes.CDLL(path)
    i32, u32, i64, sz, f32 = ctypes.c_int32, ctypes.c_uint32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    lib.pa_reshape_and_cache.argtypes = [_T, _T, _T, _T, _T, _P]
    lib.pa_copy_blocks.argtypes = [_T, _T, _T, _P]
    lib.pa_swap_blocks.argtypes = [_T, _T, _T, _T, _T, _P]
    lib.pa_prefill.argtypes = [_T, _T, _T, _T, _T, _T, _T, f32, i32, i32, _P]
    lib.pa_reshape_and_cache_fp8.argtypes = [_T, _T, _T, _T, _T, _T, _T, _P]
    lib.pa_decode_fp8.argtypes = [_T, _T, _T, _T, _T, _T, _T, _T, f32, i32, i32, i32, u32, _P, sz, _P]
    lib.pa_decode.argtypes = [_T, _T, _T, _T, _T, _T, f32, i32, i32, _P]
    lib.pa_decode_ex.argtypes = [_T, _T, _T, _T, _T, _T, f32, i32, i32, i32, u32, _P, sz, _P]
    lib.pa_decode_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
    lib.pa_decode_workspace_bytes.restype = sz
    lib.pa_decode_default_workers.argtypes = [i32, i32, i32, i32]
    lib.pa_decode_default_workers.restype = i32
    lib.pa_workspace_init.argtypes = [_P, sz, _P]
    lib.pa_release_workspaces.argtypes = []
    lib.pa_last_error.argtypes = []
    lib.pa_last_error.restype = ctypes.c_char_p
    lib.pa_get_device_error.argtypes = [_P, ctypes.POINTER(u32), i32]
    lib.pa_decode_noalloc.argtypes = [_T, _T, _T, _T, _T, _T, f32, i32, i32, _P]
    lib.pa_decode_step.argtypes = [_T, _T, _T, _T, _T, _T, _T, _T, _T, f32, i32, i32, _P, sz, _P]
    lib.pa_decode_step_fp8.argtypes = [_T] * 11 + [f32, i32, i32, _P, sz, _P]
    lib.pa_decode_step_fp8.restype = ctypes.c_int
    lib.pa_decode_shared_prefix.argtypes = [_T, _T, _T, _T, _T, _T, _T, _T, f32, i32, i32, _P, sz, _P]
    lib.pa_decode_shared_prefix.restype = ctypes.c_int
    lib.pa_decode_shared_prefix_workspace_bytes.argtypes = [i64, i32, i32, i32, i64, i32]
    lib.pa_decode_shared_prefix_workspace_bytes.restype = sz
    lib.pa_set_decode_timeline.argtypes = [_P, sz]
    lib.pa_set_decode_timeline.restype = ctypes.c_int
    lib.pa_hbm_read_probe.argtypes = [_P, sz, i32, _P, _P]
    lib.pa_hbm_read_probe.restype = ctypes.c_int
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    for name in ("pa_reshape_and_cache", "pa_copy_blocks", "pa_decode", "pa_decode_ex",
                 "pa_decode_noalloc",
                 "pa_workspace_init", "pa_release_workspaces", "pa_get_device_error"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


_DTYPE_CODES: dict = {}


def _torch_dtype_code(t) -> int:
    if not _DTYPE_CODES:
        import torch

        _DTYPE_CODES.update({torch.float32: PA_F32, torch.bfloat16: PA_BF16,
                             torch.float16: PA_F16, torch.int32: PA_I32, torch.int64: PA_I64,
                             torch.float8_e4m3fn: PA_FP8_E4M3})
    code = _DTYPE_CODES.get(t.dtype)
    if code is None:
        raise TypeError(f"unsupported tensor dtype {t.dtype}")
    return code


# A descriptor holds only the address, dtype, shape and strides, so one built for the same four
# values is the same descriptor whatever tensor they came from: descriptors are kept and reused
# (a decode loop passes the same buffers every step; building a ctypes structure costs
# microseconds of host time per tensor).
_DESCRIPTORS: dict = {}
_DESCRIPTORS_MAX = 4096


def describe(t) -> PaTensor:
    """pa_tensor descriptor of a torch tensor (no copy; the tensor must outlive the call).  The
    descriptor is shared by every tensor with the same address, dtype, shape and strides: do not
    modify it."""
    key = (t.data_ptr(), t.dtype, t.shape, t.stride())
    d = _DESCRIPTORS.get(key)
    if d is not None:
        return d
    if t.dim() > 5:
        raise ValueError("at most 5 dimensions")
    shape = (ctypes.c_int64 * 5)(*t.shape)
    stride = (ctypes.c_int64 * 5)(*t.stride())
    d = PaTensor(t.data_ptr(), _torch_dtype_code(t), t.dim(), shape, stride)
    if len(_DESCRIPTORS) >= _DESCRIPTORS_MAX:
        _DESCRIPTORS.clear()
    _DESCRIPTORS[key] = d
    return d


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(call: str, rc: int):
    if rc != PA_OK:
        raise PagedAttentionError(call, rc, (load().pa_last_error() or b"").decode())


def pa_reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, stream=None):
    """Store each new token's K/V rows at its slot (see include/pa.h)."""
    lib = load()
    d = [describe(x) for x in (key, value, key_cache, value_cache, slot_mapping)]
    _check("pa_reshape_and_cache", lib.pa_reshape_and_cache(*[ctypes.byref(x) for x in d], _stream(stream)))


def pa_copy_blocks(key_cache, value_cache, block_mapping, stream=None):
    """Copy whole blocks dst <- src for each (src, dst) row of block_mapping."""
    lib = load()
    d = [describe(x) for x in (key_cache, value_cache, block_mapping)]
    _check("pa_copy_blocks", lib.pa_copy_blocks(*[ctypes.byref(x) for x in d], _stream(stream)))


def pa_swap_blocks(src_key_cache, src_value_cache, dst_key_cache, dst_value_cache, block_mapping,
                   stream=None):
    """Move whole blocks dst <- src between two caches, e.g. device memory and pinned host
    memory (torch tensors created with pin_memory=True)."""
    lib = load()
    d = [describe(x) for x in (src_key_cache, src_value_cache, dst_key_cache, dst_value_cache,
                               block_mapping)]
    _check("pa_swap_blocks", lib.pa_swap_blocks(*[ctypes.byref(x) for x in d], _stream(stream)))


def pa_prefill(out, query, key_cache, value_cache, block_tables, context_lens, query_start, scale,
               block_size, num_kv_heads, stream=None):
    """Causal attention of each sequence's new tokens (rows query_start[s] ..
    query_start[s+1]-1, its last positions) over the paged cache (see include/pa.h)."""
    lib = load()
    d = [describe(x) for x in (out, query, key_cache, value_cache, block_tables, context_lens,
                               query_start)]
    _check("pa_prefill", lib.pa_prefill(*[ctypes.byref(x) for x in d], float(scale),
                                        int(block_size), int(num_kv_heads), _stream(stream)))


def pa_reshape_and_cache_fp8(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale,
                             stream=None):
    """Quantise new tokens' K/V rows into FP8 E4M3 caches (torch.float8_e4m3fn tensors) with
    one fp32 scale per kv head (see include/pa.h)."""
    lib = load()
    d = [describe(x) for x in (key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale)]
    _check("pa_reshape_and_cache_fp8",
           lib.pa_reshape_and_cache_fp8(*[ctypes.byref(x) for x in d], _stream(stream)))


def pa_decode_fp8(out, query, key_cache, value_cache, block_tables, context_lens, k_scale, v_scale,
                  scale, block_size, num_kv_heads, num_workers=0, flags=0, workspace=None,
                  stream=None):
    """Decode over FP8 E4M3 caches with per-kv-head scales; workspace None = library-owned."""
    lib = load()
    d = [describe(x) for x in (out, query, key_cache, value_cache, block_tables, context_lens,
                               k_scale, v_scale)]
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_fp8", lib.pa_decode_fp8(*[ctypes.byref(x) for x in d], float(scale),
                                              int(block_size), int(num_kv_heads), int(num_workers),
                                              int(flags), ws_ptr, ws_bytes, _stream(stream)))


def pa_decode(out, query, key_cache, value_cache, block_tables, context_lens, scale, block_size,
              num_kv_heads, stream=None):
    """One decode step of paged attention into `out` (library-owned workspace)."""
    lib = load()
    d = [describe(x) for x in (out, query, key_cache, value_cache, block_tables, context_lens)]
    _check("pa_decode", lib.pa_decode(*[ctypes.byref(x) for x in d], float(scale), int(block_size),
                                      int(num_kv_heads), _stream(stream)))


def pa_decode_ex(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                 block_size, num_kv_heads, num_workers=0, flags=0, workspace=None, stream=None):
    """pa_decode with an explicit warp count, flags and a caller-owned workspace (a CUDA uint8
    tensor of at least pa_decode_workspace_bytes bytes, zeroed by pa_workspace_init once)."""
    lib = load()
    d = [describe(x) for x in (out, query, key_cache, value_cache, block_tables, context_lens)]
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_ex", lib.pa_decode_ex(*[ctypes.byref(x) for x in d], float(scale),
                                            int(block_size), int(num_kv_heads), int(num_workers),
                                            int(flags), ws_ptr, ws_bytes, _stream(stream)))


def pa_decode_step_fp8(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale, out,
                       query, block_tables, context_lens, scale, block_size, num_kv_heads,
                       workspace=None, stream=None):
    """One whole step over FP8 caches: the quantising cache write and the decode, one kernel
    when each sequence brings one token in the query's type (see include/pa.h)."""
    lib = load()
    d = [describe(x) for x in (key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale,
                               out, query, block_tables, context_lens)]
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_step_fp8", lib.pa_decode_step_fp8(*[ctypes.byref(x) for x in d], float(scale),
                                                        int(block_size), int(num_kv_heads), ws_ptr,
                                                        ws_bytes, _stream(stream)))


def pa_decode_step(key, value, key_cache, value_cache, slot_mapping, out, query, block_tables,
                   context_lens, scale, block_size, num_kv_heads, workspace=None, stream=None):
    """One whole step: the cache write, then the decode launched to overlap it (see
    include/pa.h).  workspace: a CUDA uint8 tensor as for pa_decode_ex, or None for the
    library-owned one."""
    lib = load()
    d = [describe(x) for x in (key, value, key_cache, value_cache, slot_mapping, out, query,
                               block_tables, context_lens)]
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_step", lib.pa_decode_step(*[ctypes.byref(x) for x in d], float(scale),
                                                int(block_size), int(num_kv_heads), ws_ptr,
                                                ws_bytes, _stream(stream)))


def pa_decode_noalloc(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                      block_size, num_kv_heads, stream=None):
    """pa_decode for callers that cannot allocate device memory: the scratch is a fixed
    8 MiB device array inside the library (see include/pa.h); shapes that need more are
    refused with PA_ERR_WORKSPACE; calls overlapping on the GPU race on that array."""
    lib = load()
    d = [describe(x) for x in (out, query, key_cache, value_cache, block_tables, context_lens)]
    _check("pa_decode_noalloc", lib.pa_decode_noalloc(*[ctypes.byref(x) for x in d], float(scale),
                                                      int(block_size), int(num_kv_heads),
                                                      _stream(stream)))


def pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, num_workers=0) -> int:
    return int(load().pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, num_workers))


def pa_decode_default_workers(dtype: int, head_dim: int, block_size: int, group_size: int) -> int:
    return int(load().pa_decode_default_workers(dtype, head_dim, block_size, group_size))


def pa_workspace_init(workspace, stream=None):
    lib = load()
    _check("pa_workspace_init", lib.pa_workspace_init(
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream)))


def pa_release_workspaces():
    _check("pa_release_workspaces", load().pa_release_workspaces())


def pa_last_error() -> str:
    return (load().pa_last_error() or b"").decode()


def pa_get_device_error(clear: bool = False, stream=None) -> int:
    """The device error word (PA_DEVERR_* bits); synchronises the stream."""
    flags = ctypes.c_uint32(0)
    _check("pa_get_device_error", load().pa_get_device_error(_stream(stream), ctypes.byref(flags), int(clear)))
    return int(flags.value)


def pa_version() -> int:
    return int(load().pa_version())


def header_functions(path: str = HEADER) -> list[str]:
    """Names of the functions include/pa.h declares."""
    import re

    with open(path) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*PA_API\s+(?:const\s+)?\w+\s*\*?\s*(pa_\w+)\s*\(", text, re.M)))


def pa_decode_shared_prefix(out, query, key_cache, value_cache, block_tables, context_lens,
                            group_start, prefix_lens, scale, block_size, num_kv_heads,
                            workspace=None, stream=None):
    """pa_decode for groups of consecutive sequences sharing a prompt prefix (group_start
    [num_groups + 1] int32, prefix_lens [num_seqs] int32); see include/pa.h."""
    lib = load()
    d = [describe(x) for x in (out, query, key_cache, value_cache, block_tables, context_lens,
                               group_start, prefix_lens)]
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pa_decode_shared_prefix",
           lib.pa_decode_shared_prefix(*[ctypes.byref(x) for x in d], ctypes.c_float(scale),
                                       block_size, num_kv_heads, ws_ptr, ws_bytes, _stream(stream)))


def pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                            max_blocks_per_seq, block_size) -> int:
    return int(load().pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads,
                                                              head_dim, max_blocks_per_seq,
                                                              block_size))


TIMELINE_WORDS = 8  # 64-bit words per worker warp in a decode timeline record
TL_START, TL_FIRST, TL_LAST, TL_DONE, TL_SM, TL_CHUNKS, TL_ISSUE, TL_MERGED = range(8)


def pa_set_decode_timeline(buf=None):
    """Make later tensor-core decode launches record per-warp timestamps into `buf` (a CUDA
    int64 tensor, TIMELINE_WORDS words per worker warp); None stops the recording."""
    if buf is None:
        _check("pa_set_decode_timeline", load().pa_set_decode_timeline(None, 0))
    else:
        _check("pa_set_decode_timeline",
               load().pa_set_decode_timeline(buf.data_ptr(), buf.numel() * buf.element_size()))


def pa_hbm_read_probe(buf, mode: int, sink, stream=None):
    """Read every byte of the CUDA tensor `buf` once (mode 0: vector loads, 1: bulk copies into
    shared memory); `sink` is a CUDA int32 tensor of at least two elements."""
    _check("pa_hbm_read_probe",
           load().pa_hbm_read_probe(buf.data_ptr(), buf.numel() * buf.element_size(), int(mode),
                                    sink.data_ptr(), _stream(stream)))
