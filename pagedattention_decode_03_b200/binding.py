"""ctypes binding of libpa.so: same names as the C ABI (include/pa.h).

Argument marshalling only -- every step of the decode path runs in the
library's kernels; there is no CPU fallback.  torch supplies device memory
(``data_ptr()``) and streams (``torch.cuda.current_stream().cuda_stream``).
If the shared library has not been built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_NO_BLOCKS = -2
PA_ERR_NO_SEQ = -3
PA_ERR_SEQ_EXISTS = -4
PA_ERR_SHARED_BLOCK = -5
PA_ERR_CUDA = -6
PA_ERR_DEVICE_CHECK = -7

PA_BF16, PA_FP16, PA_FP8_E4M3 = 0, 1, 2
DTYPES = {"bf16": PA_BF16, "fp16": PA_FP16, "fp8_e4m3": PA_FP8_E4M3}

PA_DEVERR_BAD_BLOCK = 0x1
PA_DEVERR_BAD_LEN = 0x2
PA_DEVERR_TIMEOUT = 0x4

# every symbol include/pa.h declares
EXPORTS = (
    "pa_workspace_size", "pa_pool_create", "pa_pool_destroy", "pa_alloc_blocks",
    "pa_alloc_blocks_n", "pa_fork_cow", "pa_append_kv", "pa_decode_attention", "pa_free",
    "pa_get_seq", "pa_get_refcounts", "pa_get_free_list", "pa_get_cow_log", "pa_launch_count",
    "pa_check_device_errors", "pa_debug_fail_after", "pa_last_error", "pa_status_string",
    "pa_decode_attention_noalloc", "pa_last_decode_plan", "pa_decode_attention_append",
    "pa_plan_siblings", "pa_prefix_register", "pa_prefix_match", "pa_alloc_blocks_prefix",
    "pa_get_cached_blocks", "pa_swap_bytes", "pa_swap_out", "pa_swap_in",
    "pa_noalloc_check_errors", "pa_set_decode_path", "pa_last_decode_kernel",
    "pa_state_size", "pa_state_save", "pa_state_load",
)


class PAError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {status_string(status)} ({message})")
        self.status = status
        self.message = message


class pa_pool_desc(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("max_seqs", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32),
        ("act_dtype", ctypes.c_int32),
        ("min_partition_tokens", ctypes.c_int32),
        ("k_cache", ctypes.c_void_p),
        ("v_cache", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("k_inv_scale", ctypes.c_void_p),
        ("v_inv_scale", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("free_order", ctypes.POINTER(ctypes.c_int32)),
        ("device", ctypes.c_int32),
    ]


_lib = None
_i32p = ctypes.POINTER(ctypes.c_int32)


def lib() -> ctypes.CDLL:
    """The loaded libpa.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m pagedattention_decode_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, u32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)
        L.pa_workspace_size.argtypes = [ctypes.POINTER(pa_pool_desc)]
        L.pa_workspace_size.restype = ctypes.c_size_t
        L.pa_pool_create.argtypes = [ctypes.POINTER(pa_pool_desc), ctypes.POINTER(vp)]
        L.pa_pool_destroy.argtypes = [vp]
        L.pa_pool_destroy.restype = None
        L.pa_alloc_blocks.argtypes = [vp, i32, i32, vp]
        L.pa_alloc_blocks_n.argtypes = [vp, i32, _i32p, _i32p, vp, _i32p]
        L.pa_fork_cow.argtypes = [vp, i32, i32]
        L.pa_append_kv.argtypes = [vp, i32, i32, _i32p, _i32p, vp, vp, vp]
        L.pa_decode_attention.argtypes = [vp, i32, i32, _i32p, i32, vp, vp, ctypes.c_float, i32, vp]
        L.pa_decode_attention_append.argtypes = [vp, i32, i32, _i32p, vp, vp, i32, vp, vp, ctypes.c_float,
                                                 i32, vp]
        L.pa_decode_attention_noalloc.argtypes = [ctypes.POINTER(pa_pool_desc), i32, i32, vp, _i32p,
                                                  i32, vp, vp, ctypes.c_float, vp]
        L.pa_noalloc_check_errors.argtypes = [i32, vp, u32p]
        L.pa_noalloc_check_errors.restype = ctypes.c_int32
        L.pa_free.argtypes = [vp, i32]
        L.pa_set_decode_path.argtypes = [vp, i32]
        L.pa_set_decode_path.restype = ctypes.c_int32
        L.pa_last_decode_kernel.argtypes = [vp, _i32p]
        L.pa_last_decode_kernel.restype = ctypes.c_int32
        L.pa_prefix_register.argtypes = [vp, i32, i32, _i32p]
        L.pa_prefix_match.argtypes = [vp, i32, _i32p, _i32p]
        L.pa_alloc_blocks_prefix.argtypes = [vp, i32, i32, _i32p, _i32p]
        L.pa_get_cached_blocks.argtypes = [vp, _i32p, i32, _i32p]
        L.pa_swap_bytes.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_size_t)]
        L.pa_swap_out.argtypes = [vp, i32, vp, ctypes.c_size_t, vp]
        L.pa_swap_in.argtypes = [vp, i32, i32, vp, ctypes.c_size_t, vp]
        L.pa_get_seq.argtypes = [vp, i32, _i32p, _i32p, i32, _i32p]
        L.pa_get_refcounts.argtypes = [vp, _i32p, i32]
        L.pa_get_free_list.argtypes = [vp, _i32p, i32, _i32p]
        L.pa_get_cow_log.argtypes = [vp, _i32p, i32, _i32p]
        L.pa_launch_count.argtypes = [vp]
        L.pa_launch_count.restype = ctypes.c_uint64
        L.pa_last_decode_plan.argtypes = [vp, _i32p, ctypes.POINTER(ctypes.c_int64)]
        L.pa_plan_siblings.argtypes = [vp, i32, _i32p, i32, _i32p, _i32p, _i32p]
        L.pa_check_device_errors.argtypes = [vp, vp, u32p]
        L.pa_debug_fail_after.argtypes = [vp, i32]
        L.pa_state_size.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t)]
        L.pa_state_save.argtypes = [vp, vp, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]
        L.pa_state_load.argtypes = [vp, vp, ctypes.c_size_t]
        L.pa_last_error.argtypes = []
        L.pa_last_error.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [i32]
        L.pa_status_string.restype = ctypes.c_char_p
        for name in ("pa_pool_create", "pa_alloc_blocks", "pa_alloc_blocks_n", "pa_fork_cow",
                     "pa_decode_attention_noalloc",
                     "pa_append_kv", "pa_decode_attention", "pa_free", "pa_get_seq",
                     "pa_get_refcounts", "pa_get_free_list", "pa_get_cow_log",
                     "pa_check_device_errors", "pa_debug_fail_after"):
            getattr(L, name).restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def pa_last_error() -> str:
    return lib().pa_last_error().decode()


def pa_status_string(status: int) -> str:
    return status_string(status)


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PAError(status, where, pa_last_error())


def _i32(xs) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(xs, dtype=np.int32).reshape(-1))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_i32p)


def _stream(stream):
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        return ctypes.c_void_p(0)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Pool:
    """A pool handle plus the device buffers it points into (kept alive here)."""
    handle: ctypes.c_void_p
    desc: pa_pool_desc
    num_layers: int
    num_kv_heads: int
    block_size: int
    num_blocks: int
    max_seqs: int
    max_blocks_per_seq: int
    kv_dtype: str
    act_dtype: str
    k_cache: object = None
    v_cache: object = None
    workspace: object = None
    scales: tuple = ()
    _keep: list = field(default_factory=list)

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.pa_pool_destroy(self.handle)
            self.handle = None


def pa_workspace_size(desc: pa_pool_desc) -> int:
    return int(lib().pa_workspace_size(ctypes.byref(desc)))


def pa_pool_create(*, num_layers: int, num_kv_heads: int, block_size: int, num_blocks: int,
                   max_seqs: int, max_blocks_per_seq: int, kv_dtype: str = "bf16",
                   act_dtype: str | None = None, free_order=None, device=None,
                   k_cache=None, v_cache=None, workspace=None, k_scale=None, v_scale=None,
                   k_inv_scale=None, v_inv_scale=None, min_partition_tokens: int = 0,
                   host_only: bool = False, head_dim: int = 128) -> Pool:
    """Create a pool.  Device buffers are torch tensors (allocated here when
    not given); ``host_only=True`` makes a block-manager-only pool."""
    act_dtype = act_dtype or ("bf16" if kv_dtype == "fp8_e4m3" else kv_dtype)
    d = pa_pool_desc()
    d.num_layers, d.num_kv_heads, d.head_dim = num_layers, num_kv_heads, head_dim
    d.block_size, d.num_blocks, d.max_seqs = block_size, num_blocks, max_seqs
    d.max_blocks_per_seq = max_blocks_per_seq
    d.kv_dtype, d.act_dtype = DTYPES[kv_dtype], DTYPES[act_dtype]
    d.min_partition_tokens = min_partition_tokens
    keep = []
    if free_order is not None:
        fo = _i32(free_order)
        keep.append(fo)
        d.free_order = _ptr(fo)
    if not host_only:
        import torch
        dev = torch.device(device if device is not None else "cuda")
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        d.device = dev.index
        elem = torch.uint8 if kv_dtype == "fp8_e4m3" else (
            torch.bfloat16 if kv_dtype == "bf16" else torch.float16)
        shape = (num_layers, num_blocks, num_kv_heads, block_size, head_dim)
        if k_cache is None:
            k_cache = torch.zeros(shape, dtype=elem, device=dev)
        if v_cache is None:
            v_cache = torch.zeros(shape, dtype=elem, device=dev)
        d.k_cache, d.v_cache = k_cache.data_ptr(), v_cache.data_ptr()
        if kv_dtype == "fp8_e4m3":
            for t in (k_scale, v_scale, k_inv_scale, v_inv_scale):
                if t is None or not t.is_cuda or t.dtype != torch.float32:
                    raise ValueError("FP8 pools need fp32 device scales and inverse scales")
            d.k_scale, d.v_scale = k_scale.data_ptr(), v_scale.data_ptr()
            d.k_inv_scale, d.v_inv_scale = k_inv_scale.data_ptr(), v_inv_scale.data_ptr()
        need = pa_workspace_size(d)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        d.workspace = workspace.data_ptr()
        d.workspace_bytes = workspace.numel() * workspace.element_size()
    h = ctypes.c_void_p()
    _check(lib().pa_pool_create(ctypes.byref(d), ctypes.byref(h)), "pa_pool_create")
    return Pool(handle=h, desc=d, num_layers=num_layers, num_kv_heads=num_kv_heads,
                block_size=block_size, num_blocks=num_blocks, max_seqs=max_seqs,
                max_blocks_per_seq=max_blocks_per_seq, kv_dtype=kv_dtype, act_dtype=act_dtype,
                k_cache=k_cache, v_cache=v_cache, workspace=workspace,
                scales=(k_scale, v_scale, k_inv_scale, v_inv_scale), _keep=keep)


def pa_pool_destroy(pool: Pool) -> None:
    if pool.handle:
        lib().pa_pool_destroy(pool.handle)
        pool.handle = None


def pa_alloc_blocks(pool: Pool, seq: int, new_len: int, stream=None) -> None:
    _check(lib().pa_alloc_blocks(pool.handle, seq, new_len, _stream(stream)), "pa_alloc_blocks")


def pa_alloc_blocks_n(pool: Pool, seqs, new_lens, stream=None) -> int:
    """Reserve in order; returns how many succeeded.  On failure raises
    PAError with ``n_done`` set."""
    s, n = _i32(seqs), _i32(new_lens)
    if len(s) != len(n):
        raise ValueError("seqs and new_lens differ in length")
    done = ctypes.c_int32(0)
    st = lib().pa_alloc_blocks_n(pool.handle, len(s), _ptr(s), _ptr(n), _stream(stream),
                                 ctypes.byref(done))
    if st != PA_OK:
        err = PAError(st, "pa_alloc_blocks_n", pa_last_error())
        err.n_done = done.value
        raise err
    return done.value


def pa_fork_cow(pool: Pool, parent: int, child: int) -> None:
    _check(lib().pa_fork_cow(pool.handle, parent, child), "pa_fork_cow")


def pa_free(pool: Pool, seq: int) -> None:
    _check(lib().pa_free(pool.handle, seq), "pa_free")


def pa_prefix_register(pool: Pool, seq: int, tokens) -> None:
    """Register the full blocks of `seq` that its first len(tokens) tokens cover."""
    t = _i32(tokens)
    _check(lib().pa_prefix_register(pool.handle, seq, len(t), _ptr(t)), "pa_prefix_register")


def pa_prefix_match(pool: Pool, tokens) -> int:
    """Leading prompt tokens whose KV registered blocks hold."""
    t = _i32(tokens)
    c = ctypes.c_int32()
    _check(lib().pa_prefix_match(pool.handle, len(t), _ptr(t), ctypes.byref(c)), "pa_prefix_match")
    return c.value


def pa_alloc_blocks_prefix(pool: Pool, seq: int, tokens) -> int:
    """Create `seq` for the prompt `tokens`; returns the cached prompt tokens."""
    t = _i32(tokens)
    c = ctypes.c_int32()
    _check(lib().pa_alloc_blocks_prefix(pool.handle, seq, len(t), _ptr(t), ctypes.byref(c)),
           "pa_alloc_blocks_prefix")
    return c.value


def _dev_tensor(t, name, rows, heads, act):
    import torch
    want = torch.bfloat16 if act == "bf16" else torch.float16
    if not t.is_cuda or not t.is_contiguous() or t.dtype != want:
        raise ValueError(f"{name} must be a contiguous CUDA {act} tensor")
    if tuple(t.shape) != (rows, heads, 128):
        raise ValueError(f"{name} must have shape {(rows, heads, 128)}, got {tuple(t.shape)}")
    return t.data_ptr()


def pa_append_kv(pool: Pool, layer: int, seqs, positions, k_new, v_new, stream=None) -> None:
    s, p = _i32(seqs), _i32(positions)
    if len(s) != len(p):
        raise ValueError("seqs and positions differ in length")
    T = len(s)
    kp = _dev_tensor(k_new, "k_new", T, pool.num_kv_heads, pool.act_dtype)
    vp = _dev_tensor(v_new, "v_new", T, pool.num_kv_heads, pool.act_dtype)
    _check(lib().pa_append_kv(pool.handle, layer, T, _ptr(s), _ptr(p), ctypes.c_void_p(kp),
                              ctypes.c_void_p(vp), _stream(stream)), "pa_append_kv")


def pa_decode_attention(pool: Pool, layer: int, seqs, q, out, scale: float,
                        partition_tokens: int = 0, stream=None) -> None:
    s = _i32(seqs)
    n = len(s)
    hq = q.shape[1] if q.dim() == 3 else -1
    qp = _dev_tensor(q, "q", n, hq, pool.act_dtype)
    op = _dev_tensor(out, "out", n, hq, pool.act_dtype)
    _check(lib().pa_decode_attention(pool.handle, layer, n, _ptr(s), hq, ctypes.c_void_p(qp),
                                     ctypes.c_void_p(op), ctypes.c_float(scale),
                                     partition_tokens, _stream(stream)), "pa_decode_attention")


def pa_decode_attention_append(pool: Pool, layer: int, seqs, k_new, v_new, q, out, scale: float,
                               partition_tokens: int = 0, stream=None) -> None:
    """Append each sequence's last token (k_new/v_new [n][H_kv][128]) and decode, in one launch."""
    s = _i32(seqs)
    n = len(s)
    hq = q.shape[1] if q.dim() == 3 else -1
    kp = _dev_tensor(k_new, "k_new", n, pool.num_kv_heads, pool.act_dtype)
    vp = _dev_tensor(v_new, "v_new", n, pool.num_kv_heads, pool.act_dtype)
    qp = _dev_tensor(q, "q", n, hq, pool.act_dtype)
    op = _dev_tensor(out, "out", n, hq, pool.act_dtype)
    _check(lib().pa_decode_attention_append(pool.handle, layer, n, _ptr(s), ctypes.c_void_p(kp),
                                            ctypes.c_void_p(vp), hq, ctypes.c_void_p(qp),
                                            ctypes.c_void_p(op), ctypes.c_float(scale), partition_tokens,
                                            _stream(stream)), "pa_decode_attention_append")


def pa_decode_attention_noalloc(desc: pa_pool_desc, layer: int, block_tables, seq_lens, q, out,
                                scale: float, stream=None) -> None:
    """Decode attention without a pool or workspace (see include/pa.h): for
    callers that cannot allocate device memory.  `block_tables` is a device
    int32 tensor [n][desc.max_blocks_per_seq]; `seq_lens` host lengths [n]."""
    import torch
    lens = _i32(seq_lens)
    n = len(lens)
    if (not block_tables.is_cuda or block_tables.dtype != torch.int32 or not block_tables.is_contiguous()
            or tuple(block_tables.shape) != (n, desc.max_blocks_per_seq)):
        raise ValueError("block_tables must be a contiguous CUDA int32 tensor [n][max_blocks_per_seq]")
    act = "bf16" if desc.act_dtype == PA_BF16 else "fp16"
    hq = q.shape[1] if q.dim() == 3 else -1
    qp = _dev_tensor(q, "q", n, hq, act)
    op = _dev_tensor(out, "out", n, hq, act)
    _check(lib().pa_decode_attention_noalloc(ctypes.byref(desc), layer, n,
                                             ctypes.c_void_p(block_tables.data_ptr()), _ptr(lens), hq,
                                             ctypes.c_void_p(qp), ctypes.c_void_p(op),
                                             ctypes.c_float(scale), _stream(stream)),
           "pa_decode_attention_noalloc")


def pa_get_seq(pool: Pool, seq: int):
    """(length, block table) of `seq`."""
    L = ctypes.c_int32()
    nb = ctypes.c_int32()
    _check(lib().pa_get_seq(pool.handle, seq, ctypes.byref(L), None, 0, ctypes.byref(nb)), "pa_get_seq")
    tab = np.zeros(max(nb.value, 1), np.int32)
    _check(lib().pa_get_seq(pool.handle, seq, ctypes.byref(L), _ptr(tab), nb.value,
                            ctypes.byref(nb)), "pa_get_seq")
    return L.value, tab[: nb.value].tolist()


def pa_get_refcounts(pool: Pool):
    out = np.zeros(pool.num_blocks, np.int32)
    _check(lib().pa_get_refcounts(pool.handle, _ptr(out), pool.num_blocks), "pa_get_refcounts")
    return out.tolist()


def pa_get_free_list(pool: Pool):
    n = ctypes.c_int32()
    out = np.zeros(pool.num_blocks, np.int32)
    _check(lib().pa_get_free_list(pool.handle, _ptr(out), pool.num_blocks, ctypes.byref(n)),
           "pa_get_free_list")
    return out[: n.value].tolist()


def pa_swap_bytes(pool: Pool, n_tokens: int) -> int:
    """Bytes of the host image of an n_tokens-token sequence."""
    b = ctypes.c_size_t()
    _check(lib().pa_swap_bytes(pool.handle, n_tokens, ctypes.byref(b)), "pa_swap_bytes")
    return b.value


def _host_buffer(host):
    """(address, bytes) of a contiguous CPU torch tensor or numpy array."""
    if isinstance(host, np.ndarray):
        if not host.flags["C_CONTIGUOUS"]:
            raise ValueError("host image must be contiguous")
        return host.ctypes.data, host.nbytes
    if host.is_cuda or not host.is_contiguous():
        raise ValueError("host image must be a contiguous CPU tensor")
    return host.data_ptr(), host.numel() * host.element_size()


def pa_swap_out(pool: Pool, seq: int, host, stream=None) -> None:
    """Copy `seq`'s blocks into `host` (see pa_swap_bytes) and drop it."""
    ptr, nbytes = _host_buffer(host)
    _check(lib().pa_swap_out(pool.handle, seq, ctypes.c_void_p(ptr), nbytes, _stream(stream)),
           "pa_swap_out")


def pa_swap_in(pool: Pool, seq: int, n_tokens: int, host, stream=None) -> None:
    """Create `seq` with n_tokens tokens in fresh blocks holding the image."""
    ptr, nbytes = _host_buffer(host)
    _check(lib().pa_swap_in(pool.handle, seq, n_tokens, ctypes.c_void_p(ptr), nbytes,
                            _stream(stream)), "pa_swap_in")


def pa_get_cached_blocks(pool: Pool):
    n = ctypes.c_int32()
    out = np.zeros(pool.num_blocks, np.int32)
    _check(lib().pa_get_cached_blocks(pool.handle, _ptr(out), pool.num_blocks, ctypes.byref(n)),
           "pa_get_cached_blocks")
    return out[: n.value].tolist()


def pa_get_cow_log(pool: Pool):
    n = ctypes.c_int32()
    _check(lib().pa_get_cow_log(pool.handle, None, 0, ctypes.byref(n)), "pa_get_cow_log")
    out = np.zeros(max(2 * n.value, 2), np.int32)
    _check(lib().pa_get_cow_log(pool.handle, _ptr(out), n.value, ctypes.byref(n)), "pa_get_cow_log")
    return [(int(out[2 * k]), int(out[2 * k + 1])) for k in range(n.value)]


def pa_launch_count(pool: Pool) -> int:
    return int(lib().pa_launch_count(pool.handle))


def pa_plan_siblings(pool: Pool, seqs, group: int) -> tuple[list, list]:
    """(set of each item or -1, shared full blocks of each set) the decode would use."""
    s = _i32(seqs)
    n = len(s)
    set_of = np.zeros(max(n, 1), np.int32)
    set_cp = np.zeros(max(n, 1), np.int32)
    ns = ctypes.c_int32()
    _check(lib().pa_plan_siblings(pool.handle, n, _ptr(s), group, _ptr(set_of), _ptr(set_cp),
                                  ctypes.byref(ns)), "pa_plan_siblings")
    return set_of[:n].tolist(), set_cp[: ns.value].tolist()


def pa_last_decode_plan(pool: Pool) -> tuple[int, int]:
    """(sibling sets read once, (block, KV head) tiles read) of the last decode call."""
    sets, tiles = ctypes.c_int32(), ctypes.c_int64()
    _check(lib().pa_last_decode_plan(pool.handle, ctypes.byref(sets), ctypes.byref(tiles)),
           "pa_last_decode_plan")
    return sets.value, tiles.value


def pa_check_device_errors(pool: Pool, stream=None) -> int:
    """Synchronise, read and clear the device error word; returns its bits
    (raises PAError only for CUDA failures)."""
    bits = ctypes.c_uint32(0)
    st = lib().pa_check_device_errors(pool.handle, _stream(stream), ctypes.byref(bits))
    if st not in (PA_OK, PA_ERR_DEVICE_CHECK):
        _check(st, "pa_check_device_errors")
    return bits.value


PA_DECODE_AUTO, PA_DECODE_WARP, PA_DECODE_TCGEN05 = 0, 1, 2
DECODE_PATHS = {"auto": PA_DECODE_AUTO, "warp": PA_DECODE_WARP, "tcgen05": PA_DECODE_TCGEN05}


def pa_set_decode_path(pool: Pool, path) -> None:
    """Kernel for a query group of 8 over 16-bit KV: "auto", "warp" or "tcgen05"."""
    _check(lib().pa_set_decode_path(pool.handle, DECODE_PATHS.get(path, path)), "pa_set_decode_path")


def pa_last_decode_kernel(pool: Pool) -> str:
    """"tcgen05" if the last decode call ran the tcgen05 kernel, else "warp"."""
    v = ctypes.c_int32()
    _check(lib().pa_last_decode_kernel(pool.handle, ctypes.byref(v)), "pa_last_decode_kernel")
    return "tcgen05" if v.value else "warp"


def pa_noalloc_check_errors(device: int = 0, stream=None) -> int:
    """Synchronise, read and clear the error word of the no-allocation
    scratch on `device`; returns its bits (raises PAError only for CUDA
    failures)."""
    bits = ctypes.c_uint32(0)
    st = lib().pa_noalloc_check_errors(device, _stream(stream), ctypes.byref(bits))
    if st not in (PA_OK, PA_ERR_DEVICE_CHECK):
        _check(st, "pa_noalloc_check_errors")
    return bits.value


def pa_debug_fail_after(pool: Pool, n: int) -> None:
    _check(lib().pa_debug_fail_after(pool.handle, n), "pa_debug_fail_after")


def pa_state_size(pool: Pool) -> int:
    n = ctypes.c_size_t()
    _check(lib().pa_state_size(pool.handle, ctypes.byref(n)), "pa_state_size")
    return int(n.value)


def pa_state_save(pool: Pool) -> bytes:
    """The pool's host state image (pa.h: host state checkpoint)."""
    buf = ctypes.create_string_buffer(pa_state_size(pool))
    n = ctypes.c_size_t()
    _check(lib().pa_state_save(pool.handle, buf, len(buf), ctypes.byref(n)), "pa_state_save")
    return buf.raw[: n.value]


def pa_state_load(pool: Pool, image: bytes) -> None:
    buf = ctypes.create_string_buffer(bytes(image), len(image))
    _check(lib().pa_state_load(pool.handle, buf, len(image)), "pa_state_load")
