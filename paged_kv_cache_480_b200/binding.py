"""ctypes binding of libpagedkv.so: argument marshalling only.

Every function takes torch tensors (device memory and streams come from
PyTorch), checks their placement and dtype, and passes raw pointers and sizes
to the C ABI declared in ``include/pagedkv.h``.  All arithmetic runs in the
library's CUDA kernels; if the library is missing, calls raise.
"""
import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpagedkv.so")

PKV_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
          4: "out of blocks", 5: "unknown or duplicate sequence id", 6: "workspace too small",
          7: "a device-side check fired"}
DEVERR = {1: "block id out of range", 2: "slot out of range", 4: "context length out of range",
          8: "copy pair out of range", 16: "bounded wait gave up", 32: "copy pairs overlap"}


class PagedKVError(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class OutOfBlocks(PagedKVError):
    pass


_lib = None
_lock = threading.Lock()


def load_library(path=LIB_PATH):
    """Open libpagedkv.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise FileNotFoundError(
                f"{path} is missing: build it with `python -m paged_kv_cache_480_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        lib.pkv_status_string.argtypes = [I]
        lib.pkv_status_string.restype = ctypes.c_char_p
        lib.pkv_version.restype = ctypes.c_char_p
        lib.paged_attention_decode.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, P, SZ, P]
        lib.paged_attention_decode.restype = I
        lib.paged_attention_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        lib.paged_attention_workspace_size.restype = SZ
        lib.paged_attention_partition_size.argtypes = [I, I, I, I, I]
        lib.paged_attention_partition_size.restype = I
        lib.paged_attention_workspace_init.argtypes = [P, SZ, P]
        lib.paged_attention_workspace_init.restype = I
        lib.reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I64, I64, I, P]
        lib.reshape_and_cache.restype = I
        lib.copy_blocks.argtypes = [P, P, I, P, I, I, I64, P]
        lib.copy_blocks.restype = I
        lib.paged_attention_decode_append.argtypes = [P, P, P, P, P, P, P, P, P, F, I, I, I, I, I, I, I, I,
                                                      I64, I64, I, I, P, SZ, P]
        lib.paged_attention_decode_append.restype = I
        lib.paged_attention_decode_noalloc.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, P]
        lib.paged_attention_decode_noalloc.restype = I
        lib.swap_blocks.argtypes = [P, P, I, P, I, I, I, I64, P]
        lib.swap_blocks.restype = I
        lib.pkv_bm_swap_out.argtypes = [P, P, I64, P, I, ctypes.POINTER(I)]
        lib.pkv_bm_swap_out.restype = I
        lib.paged_attention_decode_fp8kv.argtypes = [P, P, P, P, P, P, F, F, F, I, I, I, I, I, I, I, I,
                                                     I, I, P, SZ, P]
        lib.paged_attention_decode_fp8kv.restype = I
        lib.reshape_and_cache_fp8kv.argtypes = [P, P, P, P, P, I, I, I, I, I, I64, I64, I, F, F, P]
        lib.reshape_and_cache_fp8kv.restype = I
        lib.paged_attention_prefill.argtypes = [P, P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, I, P]
        lib.paged_attention_prefill.restype = I
        lib.pkv_read_device_errors.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
        lib.pkv_read_device_errors.restype = I
        lib.pkv_set_wait_limit.argtypes = [I64]
        lib.pkv_set_wait_limit.restype = I
        lib.pkv_bm_create.argtypes = [I, I, P, ctypes.POINTER(P)]
        lib.pkv_bm_create.restype = I
        lib.pkv_bm_destroy.argtypes = [P]
        lib.pkv_bm_destroy.restype = None
        lib.pkv_bm_allocate.argtypes = [P, I64, I]
        lib.pkv_bm_allocate.restype = I
        lib.pkv_bm_fork.argtypes = [P, I64, I64]
        lib.pkv_bm_fork.restype = I
        lib.pkv_bm_append_slot.argtypes = [P, I64, ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int32)]
        lib.pkv_bm_append_slot.restype = I
        lib.pkv_bm_append_slots.argtypes = [P, P, I, P, P, ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.pkv_bm_append_slots.restype = I
        lib.pkv_bm_free.argtypes = [P, I64]
        lib.pkv_bm_free.restype = I
        lib.pkv_bm_block_table.argtypes = [P, I64, P, I, ctypes.POINTER(I)]
        lib.pkv_bm_block_table.restype = I
        lib.pkv_bm_fill_tables.argtypes = [P, P, I, P, I, P]
        lib.pkv_bm_fill_tables.restype = I
        lib.pkv_bm_num_free.argtypes = [P]
        lib.pkv_bm_num_free.restype = I
        lib.pkv_bm_seq_len.argtypes = [P, I64]
        lib.pkv_bm_seq_len.restype = I
        lib.pkv_bm_ref_count.argtypes = [P, ctypes.c_int32]
        lib.pkv_bm_ref_count.restype = I
        lib.pkv_bm_utilisation.argtypes = [P]
        lib.pkv_bm_utilisation.restype = ctypes.c_double
        _lib = lib
        return lib


def _check(status, what):
    if status != PKV_OK:
        raise (OutOfBlocks if status == 4 else PagedKVError)(status, what)


def _dtype_code(t):
    import torch
    codes = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _stream(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _contig(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return _cuda(t, name)


# ---------------------------------------------------------------------------
# workspace: one zero-initialised buffer per device, grown on demand
# ---------------------------------------------------------------------------
_workspaces = {}


def default_workspace(device, nbytes):
    """The binding's per-device workspace (not for concurrent streams)."""
    import torch
    idx = device.index if device.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(idx)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _workspaces[idx] = ws
    return ws


def paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_size, block_size,
                                   max_context_len, dtype_code, partition_size=0):
    return load_library().paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                         head_size, block_size, max_context_len,
                                                         dtype_code, partition_size)


def paged_attention_partition_size(num_heads, num_kv_heads, block_size, max_context_len,
                                   partition_size=0):
    return load_library().paged_attention_partition_size(num_heads, num_kv_heads, block_size,
                                                         max_context_len, partition_size)


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                           num_kv_heads=None, block_size=None, max_context_len=None,
                           partition_size=0, workspace=None, stream=None):
    """Decode attention through the block table (see paged_attention_decode in pagedkv.h).

    out, q: [S, H, D]; k_cache, v_cache: [NB, Hkv, bs, D]; block_tables: int32
    [S, MB]; context_lens: int32 [S].  ``max_context_len`` defaults to MB *
    bs (no host/device synchronisation).
    """
    import torch
    lib = load_library()
    S, H, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if num_kv_heads is None:
        num_kv_heads = Hkv
    if block_size is None:
        block_size = bs
    if (num_kv_heads, block_size, D) != (Hkv, bs, D2) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache shape does not match num_kv_heads / block_size / head_size")
    if out.shape != q.shape or out.dtype != q.dtype or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("out, q and the caches must share shape/dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    MB = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = MB * bs
    code = _dtype_code(q)
    need = lib.paged_attention_workspace_size(S, H, Hkv, D, bs, max_context_len, code, partition_size)
    if need == 0:
        raise PagedKVError(2, "paged_attention_workspace_size")
    if workspace is None:
        workspace = default_workspace(q.device, need)
    st = lib.paged_attention_decode(
        _contig(out, "out"), _contig(q, "q"), _contig(k_cache, "k_cache"), _contig(v_cache, "v_cache"),
        _contig(block_tables, "block_tables"), _contig(context_lens, "context_lens"),
        float(scale), Hkv, bs, S, H, D, NB, MB, int(max_context_len), code, int(partition_size),
        _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream, q.device))
    _check(st, "paged_attention_decode")
    return out


def paged_attention_decode_append(out, q, key, value, k_cache, v_cache, slot_mapping,
                                  block_tables, context_lens, scale, max_context_len=None,
                                  partition_size=0, workspace=None, stream=None):
    """reshape_and_cache of one new token per sequence fused into the decode
    (paged_attention_decode_append in pagedkv.h).  key/value: [S, Hkv, D]
    (token stride may exceed Hkv * D); slot_mapping: int64 [S], each the slot
    of position context_lens[s] - 1, or negative for none."""
    import torch
    lib = load_library()
    S, H, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if tuple(key.shape) != (S, Hkv, D) or tuple(value.shape) != (S, Hkv, D):
        raise ValueError("key/value must be [num_seqs, num_kv_heads, head_size]")
    if key.stride(2) != 1 or key.stride(1) != D or value.stride(2) != 1 or value.stride(1) != D:
        raise ValueError("key/value heads must be contiguous within a token")
    for t in (key, value, k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise ValueError("all tensors must share q's dtype")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != S:
        raise TypeError("slot_mapping must be int64 [num_seqs]")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    MB = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = MB * bs
    code = _dtype_code(q)
    need = lib.paged_attention_workspace_size(S, H, Hkv, D, bs, max_context_len, code, partition_size)
    if need == 0:
        raise PagedKVError(2, "paged_attention_workspace_size")
    if workspace is None:
        workspace = default_workspace(q.device, need)
    st = lib.paged_attention_decode_append(
        _contig(out, "out"), _contig(q, "q"), _cuda(key, "key"), _cuda(value, "value"),
        _contig(k_cache, "k_cache"), _contig(v_cache, "v_cache"), _contig(slot_mapping, "slot_mapping"),
        _contig(block_tables, "block_tables"), _contig(context_lens, "context_lens"), float(scale),
        Hkv, bs, S, H, D, NB, MB, int(max_context_len), key.stride(0), value.stride(0), code,
        int(partition_size), _cuda(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream, q.device))
    _check(st, "paged_attention_decode_append")
    return out


def _fp8_cache(t, name):
    import torch
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn)")
    return _contig(t, name)


def paged_attention_decode_fp8kv(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                 k_scale, v_scale, max_context_len=None, partition_size=0,
                                 workspace=None, stream=None):
    """Decode attention over FP8 E4M3 caches (paged_attention_decode_fp8kv in
    pagedkv.h): k_cache / v_cache uint8 [NB, Hkv, bs, D]; q, out in f32/f16/bf16."""
    import torch
    lib = load_library()
    S, H, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("shape / dtype mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    MB = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = MB * bs
    code = _dtype_code(q)
    need = lib.paged_attention_workspace_size(S, H, Hkv, D, bs, max_context_len, code, partition_size)
    if need == 0:
        raise PagedKVError(2, "paged_attention_workspace_size")
    if workspace is None:
        workspace = default_workspace(q.device, need)
    st = lib.paged_attention_decode_fp8kv(
        _contig(out, "out"), _contig(q, "q"), _fp8_cache(k_cache, "k_cache"), _fp8_cache(v_cache, "v_cache"),
        _contig(block_tables, "block_tables"), _contig(context_lens, "context_lens"), float(scale),
        float(k_scale), float(v_scale), Hkv, bs, S, H, D, NB, MB, int(max_context_len), code,
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream, q.device))
    _check(st, "paged_attention_decode_fp8kv")
    return out


def paged_attention_prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                            scale, max_query_len=None, stream=None):
    """Causal prefill / chunked-prefill attention over the paged cache
    (paged_attention_prefill in pagedkv.h): q, out [T, H, D] packed by
    sequence (query_start_loc int32 [S + 1]); the last n_s tokens of each
    sequence's context_lens[s] cached tokens are its queries."""
    import torch
    lib = load_library()
    T, H, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if out.dtype != q.dtype or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise TypeError("q, caches and out must share one dtype")
    if (block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32
            or query_start_loc.dtype != torch.int32):
        raise TypeError("block_tables, context_lens and query_start_loc must be int32")
    S = context_lens.numel()
    if query_start_loc.numel() != S + 1 or block_tables.shape[0] != S:
        raise ValueError("query_start_loc must be [S + 1] and block_tables [S, MB]")
    if max_query_len is None:
        raise ValueError("max_query_len is required (a host-known bound of the queries per sequence)")
    st = lib.paged_attention_prefill(
        _contig(out, "out"), _contig(q, "q"), _contig(k_cache, "k_cache"), _contig(v_cache, "v_cache"),
        _contig(block_tables, "block_tables"), _contig(context_lens, "context_lens"),
        _contig(query_start_loc, "query_start_loc"), float(scale), T, S, H, Hkv, D, bs, NB,
        block_tables.shape[1], int(max_query_len), _dtype_code(q), _stream(stream, q.device))
    _check(st, "paged_attention_prefill")
    return out


def reshape_and_cache_fp8kv(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale, stream=None):
    """Quantising cache write into FP8 E4M3 caches (reshape_and_cache_fp8kv in pagedkv.h)."""
    import torch
    lib = load_library()
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv, D) != (Hkv2, D2) or value.shape != key.shape:
        raise ValueError("key/value shape does not match the cache")
    if key.stride(2) != 1 or key.stride(1) != D or value.stride(2) != 1 or value.stride(1) != D:
        raise ValueError("key/value heads must be contiguous within a token")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != T:
        raise TypeError("slot_mapping must be int64 [T]")
    st = lib.reshape_and_cache_fp8kv(
        _cuda(key, "key"), _cuda(value, "value"), _fp8_cache(k_cache, "k_cache"),
        _fp8_cache(v_cache, "v_cache"), _contig(slot_mapping, "slot_mapping"), T, Hkv, D, bs, NB,
        key.stride(0), value.stride(0), _dtype_code(key), float(k_scale), float(v_scale),
        _stream(stream, key.device))
    _check(st, "reshape_and_cache_fp8kv")


NOALLOC_SCRATCH_BYTES = 16 << 20


def paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                   max_context_len=None, partition_size=0, stream=None):
    """Decode attention using the library's fixed internal scratch instead of
    a workspace (paged_attention_decode_noalloc in pagedkv.h): for callers
    that cannot allocate device memory.  Calls on different streams must not
    overlap; sizes needing more than 16 MiB of scratch raise."""
    import torch
    lib = load_library()
    S, H, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if out.dtype != q.dtype or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("out, q and the caches must share a dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    MB = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = MB * bs
    st = lib.paged_attention_decode_noalloc(
        _contig(out, "out"), _contig(q, "q"), _contig(k_cache, "k_cache"), _contig(v_cache, "v_cache"),
        _contig(block_tables, "block_tables"), _contig(context_lens, "context_lens"),
        float(scale), Hkv, bs, S, H, D, NB, MB, int(max_context_len), _dtype_code(q),
        int(partition_size), _stream(stream, q.device))
    _check(st, "paged_attention_decode_noalloc")
    return out


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """Write key/value rows [T, Hkv, D] (token stride may exceed Hkv * D) into their slots."""
    import torch
    lib = load_library()
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv, D) != (Hkv2, D2) or value.shape != key.shape:
        raise ValueError("key/value shape does not match the cache")
    if key.stride(2) != 1 or key.stride(1) != D or value.stride(2) != 1 or value.stride(1) != D:
        raise ValueError("key/value heads must be contiguous within a token")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != T:
        raise TypeError("slot_mapping must be int64 [T]")
    if key.dtype != k_cache.dtype or value.dtype != v_cache.dtype or k_cache.dtype != v_cache.dtype:
        raise ValueError("dtype mismatch")
    st = lib.reshape_and_cache(
        _cuda(key, "key"), _cuda(value, "value"), _contig(k_cache, "k_cache"),
        _contig(v_cache, "v_cache"), _contig(slot_mapping, "slot_mapping"), T, Hkv, D, bs, NB,
        key.stride(0), value.stride(0), _dtype_code(key), _stream(stream, key.device))
    _check(st, "reshape_and_cache")


def copy_blocks(k_caches, v_caches, block_mapping, stream=None):
    """Copy-on-write block copies: block_mapping int64 [N, 2] (src, dst) on the device."""
    import torch
    lib = load_library()
    if len(k_caches) != len(v_caches) or not k_caches:
        raise ValueError("need matching non-empty lists of caches")
    if block_mapping.dtype != torch.int64:
        raise TypeError("block_mapping must be int64")
    NB = k_caches[0].shape[0]
    block_bytes = k_caches[0][0].numel() * k_caches[0].element_size()
    for c in list(k_caches) + list(v_caches):
        if c.shape != k_caches[0].shape or c.dtype != k_caches[0].dtype:
            raise ValueError("all caches must share shape and dtype")
    n = len(k_caches)
    karr = (ctypes.c_void_p * n)(*[_contig(c, "k_cache").value for c in k_caches])
    varr = (ctypes.c_void_p * n)(*[_contig(c, "v_cache").value for c in v_caches])
    pairs = block_mapping.numel() // 2
    st = lib.copy_blocks(karr, varr, n, _contig(block_mapping, "block_mapping"), pairs, NB,
                         block_bytes, _stream(stream, k_caches[0].device))
    _check(st, "copy_blocks")


def swap_blocks(src_caches, dst_caches, block_mapping, stream=None):
    """Block copies between two pools (device or pinned host memory), e.g. the
    K and V caches of every layer: dst_caches[c][dst] = src_caches[c][src]
    for each (src, dst) row of block_mapping (int64 [N, 2], device or pinned)."""
    import torch
    lib = load_library()
    if len(src_caches) != len(dst_caches) or not src_caches:
        raise ValueError("need matching non-empty lists of caches")
    if block_mapping.dtype != torch.int64:
        raise TypeError("block_mapping must be int64")
    block_bytes = src_caches[0][0].numel() * src_caches[0].element_size()
    for c in list(src_caches) + list(dst_caches):
        if c[0].numel() * c.element_size() != block_bytes or not c.is_contiguous():
            raise ValueError("all pools must be contiguous with equal block sizes")
    n = len(src_caches)
    sarr = (ctypes.c_void_p * n)(*[c.data_ptr() for c in src_caches])
    darr = (ctypes.c_void_p * n)(*[c.data_ptr() for c in dst_caches])
    dev = next((c.device for c in list(src_caches) + list(dst_caches) if c.is_cuda), None)
    s = _stream(stream, dev) if dev is not None else ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.swap_blocks(sarr, darr, n, ctypes.c_void_p(block_mapping.data_ptr()),
                         block_mapping.numel() // 2, src_caches[0].shape[0], dst_caches[0].shape[0],
                         block_bytes, s)
    _check(st, "swap_blocks")


def read_device_errors(stream=None):
    """Synchronise the stream and return (and clear) the sticky device-check bits."""
    import torch
    lib = load_library()
    bits = ctypes.c_uint32(0)
    s = ctypes.c_void_p(stream.cuda_stream) if stream is not None else \
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.pkv_read_device_errors(s, ctypes.byref(bits))
    if st not in (0, 7):
        _check(st, "pkv_read_device_errors")
    return bits.value


def set_wait_limit(polls):
    """For tests of the failure path: polls after which the kernels' bounded
    waits give up (pkv_set_wait_limit in pagedkv.h); negative restores the
    default."""
    _check(load_library().pkv_set_wait_limit(int(polls)), "pkv_set_wait_limit")


class BlockManager:
    """Host block manager (pkv_bm_* in pagedkv.h)."""

    def __init__(self, num_blocks, block_size, free_order=None):
        import numpy as np
        self._lib = load_library()
        self.block_size = block_size
        self.num_blocks = num_blocks
        h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(free_order, dtype=np.int32)
            order = ctypes.c_void_p(self._order.ctypes.data)
        _check(self._lib.pkv_bm_create(num_blocks, block_size, order, ctypes.byref(h)), "pkv_bm_create")
        self._h = h

    def close(self):
        if self._h:
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, seq, num_tokens):
        _check(self._lib.pkv_bm_allocate(self._h, seq, num_tokens), "pkv_bm_allocate")

    def fork(self, parent, child):
        _check(self._lib.pkv_bm_fork(self._h, parent, child), "pkv_bm_fork")

    def append_slot(self, seq):
        slot = ctypes.c_int64()
        src, dst = ctypes.c_int32(), ctypes.c_int32()
        _check(self._lib.pkv_bm_append_slot(self._h, seq, ctypes.byref(slot), ctypes.byref(src),
                                            ctypes.byref(dst)), "pkv_bm_append_slot")
        return slot.value, (None if src.value < 0 else (src.value, dst.value))

    def append_slots(self, seq_ids):
        """Slots (int64 [n]) and CoW pairs (int64 [k, 2]) for one token per sequence."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        slots = np.empty(len(ids), np.int64)
        pairs = np.empty((max(len(ids), 1), 2), np.int64)
        ncow, ndone = ctypes.c_int(), ctypes.c_int()
        st = self._lib.pkv_bm_append_slots(self._h, ids.ctypes.data, len(ids), slots.ctypes.data,
                                           pairs.ctypes.data, ctypes.byref(ncow), ctypes.byref(ndone))
        _check(st, "pkv_bm_append_slots")
        return slots, pairs[:ncow.value].copy()

    def free(self, seq):
        _check(self._lib.pkv_bm_free(self._h, seq), "pkv_bm_free")

    def swap_out(self, host, seq):
        """Move sequence seq to manager `host` (all or nothing); returns int64
        [n, 2] (block here, block in host) pairs for swap_blocks.  Swapping
        back in is host.swap_out(self, seq)."""
        import numpy as np
        cap = max(self.num_blocks, host.num_blocks)
        pairs = np.empty((cap, 2), np.int64)
        n = ctypes.c_int()
        st = self._lib.pkv_bm_swap_out(self._h, host._h, seq, pairs.ctypes.data, cap, ctypes.byref(n))
        _check(st, "pkv_bm_swap_out")
        return pairs[:n.value].copy()

    def block_table(self, seq):
        import numpy as np
        n = ctypes.c_int()
        _check(self._lib.pkv_bm_block_table(self._h, seq, None, 0, ctypes.byref(n)), "pkv_bm_block_table")
        out = np.empty(max(n.value, 1), np.int32)
        _check(self._lib.pkv_bm_block_table(self._h, seq, out.ctypes.data, n.value, ctypes.byref(n)),
               "pkv_bm_block_table")
        return out[:n.value]

    def fill_tables(self, seq_ids, max_blocks_per_seq):
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.empty((len(ids), max_blocks_per_seq), np.int32)
        lens = np.empty(len(ids), np.int32)
        _check(self._lib.pkv_bm_fill_tables(self._h, ids.ctypes.data, len(ids), tables.ctypes.data,
                                            max_blocks_per_seq, lens.ctypes.data), "pkv_bm_fill_tables")
        return tables, lens

    def num_free(self):
        return self._lib.pkv_bm_num_free(self._h)

    def seq_len(self, seq):
        return self._lib.pkv_bm_seq_len(self._h, seq)

    def ref_count(self, block):
        return self._lib.pkv_bm_ref_count(self._h, block)

    def utilisation(self):
        return self._lib.pkv_bm_utilisation(self._h)
