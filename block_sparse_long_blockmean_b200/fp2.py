"""ctypes binding of ``libfp2.so`` (include/fp2.h), with the same names.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are passed by ``data_ptr()``; the stream defaults to
torch's current stream.  PyTorch is used for device memory and streams.
There is no fallback: if the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp2.so")

FP2_OK = 0
FP2_ERR_INVALID_ARG = 1
FP2_ERR_UNSUPPORTED = 2
FP2_ERR_WORKSPACE = 3
FP2_ERR_CUDA = 4
FP2_ERR_TIMEOUT = 5
FP2_ERR_DEVICE_BOUNDS = 6

FP2_BF16 = 0
FP2_FP8_E4M3 = 1


class Fp2Error(RuntimeError):
    def __init__(self, status: int, where: str, detail: int = 0):
        self.status = status
        self.detail = detail
        msg = status_string(status) if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status}, detail {detail})")


class Params(ctypes.Structure):
    """Mirror of ``fp2_params``."""
    _fields_ = [
        ("num_seqs", ctypes.c_int),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("total_q", ctypes.c_int),
        ("total_k", ctypes.c_int),
        ("page_size", ctypes.c_int),
        ("max_pages_per_seq", ctypes.c_int),
        ("num_pages", ctypes.c_int),
        ("max_seqlen_q", ctypes.c_int),
        ("max_seqlen_k", ctypes.c_int),
        ("seqlens_k", ctypes.c_void_p),
        ("cu_seqlens_k", ctypes.c_void_p),
        ("q_scale", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p),
        ("group_masks", ctypes.c_int),
        ("out_dtype", ctypes.c_int),
        ("out_scale", ctypes.c_void_p),
        ("attn_kernel", ctypes.c_int),
        ("debug_wait_limit_us", ctypes.c_uint),
        ("debug_withhold_k_item", ctypes.c_int),
        ("k_block_factor", ctypes.c_void_p),
        ("v_block_factor", ctypes.c_void_p),
    ]


class WorkspaceLayout(ctypes.Structure):
    """Mirror of ``fp2_workspace_layout``."""
    _fields_ = [
        ("error_word", ctypes.c_size_t),
        ("kbar", ctypes.c_size_t),
        ("vbar", ctypes.c_size_t),
        ("kbar_op", ctypes.c_size_t),
        ("vbar_op", ctypes.c_size_t),
        ("scores", ctypes.c_size_t),
        ("kept_idx", ctypes.c_size_t),
        ("kept_cnt", ctypes.c_size_t),
        ("kept_bits", ctypes.c_size_t),
        ("total", ctypes.c_size_t),
        ("nqb_max", ctypes.c_int),
        ("nkb_max", ctypes.c_int),
        ("nw", ctypes.c_int),
    ]


class HostIO(ctypes.Structure):
    """Mirror of ``fp2_host_io`` (host buffers, their device twins, the copy
    streams and the number of query-block chunks of fp2_prefill_host)."""
    _fields_ = [
        ("q_host", ctypes.c_void_p),
        ("k_host", ctypes.c_void_p),
        ("v_host", ctypes.c_void_p),
        ("out_host", ctypes.c_void_p),
        ("q_dev", ctypes.c_void_p),
        ("k_dev", ctypes.c_void_p),
        ("v_dev", ctypes.c_void_p),
        ("out_dev", ctypes.c_void_p),
        ("cu_seqlens_host", ctypes.c_void_p),
        ("seqlens_k_host", ctypes.c_void_p),
        ("cu_seqlens_k_host", ctypes.c_void_p),
        ("upload_stream", ctypes.c_void_p),
        ("download_stream", ctypes.c_void_p),
        ("num_chunks", ctypes.c_int),
    ]


_LIB = None
_VP = ctypes.c_void_p
_PP = ctypes.POINTER(Params)

# name -> (restype, argtypes); the exported C-ABI
SIGNATURES = {
    "fp2_workspace_size": (ctypes.c_size_t, [_PP, ctypes.c_int]),
    "fp2_get_workspace_layout": (ctypes.c_int, [_PP, ctypes.c_int, ctypes.POINTER(WorkspaceLayout)]),
    "fp2_prefill": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, ctypes.c_float, ctypes.c_int,
                                   ctypes.c_int, _VP, _PP]),
    "fp2_prefill_noalloc": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, ctypes.c_float, ctypes.c_int,
                                           ctypes.c_int, _VP, _PP]),
    "fp2_prefill_cached": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_int, _VP, _PP, _VP, ctypes.c_int, _VP,
                                          ctypes.c_int]),
    "fp2_prefill_host": (ctypes.c_int, [ctypes.POINTER(HostIO), _VP, _VP, ctypes.c_float,
                                        ctypes.c_int, ctypes.c_int, _PP]),
    "fp2_blockmean": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, ctypes.c_int, _PP]),
    "fp2_blockmean_cached": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, ctypes.c_int, _VP,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, _PP]),
    "fp2_score": (ctypes.c_int, [_VP, _VP, ctypes.c_int, ctypes.c_int, _PP]),
    "fp2_mask": (ctypes.c_int, [_VP, ctypes.c_float, ctypes.c_int, _PP]),
    "fp2_attn": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int, ctypes.c_int, _VP,
                                _PP]),
    "fp2_workspace_init": (ctypes.c_int, [_PP]),
    "fp2_get_status": (ctypes.c_int, [_PP, ctypes.POINTER(ctypes.c_uint32)]),
    "fp2_noalloc_get_status": (ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_uint32)]),
    "fp2_calibrate_tau": (ctypes.c_int, [_VP, ctypes.c_int, ctypes.c_float, _PP,
                                         ctypes.POINTER(ctypes.c_float)]),
    "fp2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fp2_version": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it was not built (no fallback)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_long_blockmean_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = h
    return _LIB


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _check(st: int, where: str):
    if st != FP2_OK:
        raise Fp2Error(st, where)


def status_string(st: int) -> str:
    return lib().fp2_status_string(st).decode()


def version() -> str:
    return lib().fp2_version().decode()


def workspace_size(params: Params, block: int) -> int:
    return int(lib().fp2_workspace_size(ctypes.byref(params), block))


def get_workspace_layout(params: Params, block: int) -> WorkspaceLayout:
    L = WorkspaceLayout()
    _check(lib().fp2_get_workspace_layout(ctypes.byref(params), block, ctypes.byref(L)),
           "fp2_get_workspace_layout")
    return L


def prefill(q, k_cache, v_cache, page_table, cu_seqlens, tau: float, block: int, dtype: int,
            out, params: Params) -> None:
    _check(lib().fp2_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                             _ptr(cu_seqlens), float(tau), block, dtype, _ptr(out),
                             ctypes.byref(params)), "fp2_prefill")


def prefill_noalloc(q, k_cache, v_cache, page_table, cu_seqlens, tau: float, block: int,
                    dtype: int, out, params: Params) -> None:
    """fp2_prefill with library-owned scratch (params.workspace is ignored)."""
    _check(lib().fp2_prefill_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                     _ptr(cu_seqlens), float(tau), block, dtype, _ptr(out),
                                     ctypes.byref(params)), "fp2_prefill_noalloc")


def prefill_host(io: HostIO, page_table, cu_seqlens, tau: float, block: int, dtype: int,
                 params: Params) -> None:
    """fp2_prefill with q, K/V and out in (pinned) host memory, copies
    pipelined with the kernels over ``io.num_chunks`` query-block ranges.
    ``io`` holds raw pointers; the caller keeps the tensors behind them alive
    until ``params.stream`` has been synchronised."""
    _check(lib().fp2_prefill_host(ctypes.byref(io), _ptr(page_table), _ptr(cu_seqlens),
                                  float(tau), block, dtype, ctypes.byref(params)),
           "fp2_prefill_host")


def host_io(q_host, k_host, v_host, out_host, q_dev, k_dev, v_dev, out_dev, cu_seqlens_host,
            seqlens_k_host=None, upload_stream=None, download_stream=None,
            num_chunks: int = 16, cu_seqlens_k_host=None) -> HostIO:
    """An ``fp2_host_io`` from tensors (host ones on the CPU, ideally pinned;
    int32 length arrays on the CPU) and torch streams (or None)."""
    io = HostIO()
    io.q_host, io.k_host, io.v_host, io.out_host = (_ptr(q_host), _ptr(k_host), _ptr(v_host),
                                                    _ptr(out_host))
    io.q_dev, io.k_dev, io.v_dev, io.out_dev = _ptr(q_dev), _ptr(k_dev), _ptr(v_dev), _ptr(out_dev)
    io.cu_seqlens_host = _ptr(cu_seqlens_host)
    io.seqlens_k_host = _ptr(seqlens_k_host)
    io.cu_seqlens_k_host = _ptr(cu_seqlens_k_host)
    io.upload_stream = upload_stream.cuda_stream if upload_stream is not None else None
    io.download_stream = download_stream.cuda_stream if download_stream is not None else None
    io.num_chunks = int(num_chunks)
    return io


def blockmean(k_cache, v_cache, page_table, cu_seqlens, block: int, dtype: int,
              params: Params) -> None:
    _check(lib().fp2_blockmean(_ptr(k_cache), _ptr(v_cache), _ptr(page_table), _ptr(cu_seqlens),
                               block, dtype, ctypes.byref(params)), "fp2_blockmean")


def prefill_cached(q, k_cache, v_cache, page_table, cu_seqlens, tau: float, block: int,
                   dtype: int, out, params: Params, block_table, max_blocks_per_seq: int,
                   mean_cache, num_slots: int) -> None:
    _check(lib().fp2_prefill_cached(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                    _ptr(cu_seqlens), float(tau), block, dtype, _ptr(out),
                                    ctypes.byref(params), _ptr(block_table), max_blocks_per_seq,
                                    _ptr(mean_cache), num_slots), "fp2_prefill_cached")


def blockmean_cached(k_cache, v_cache, page_table, cu_seqlens, block_table,
                     max_blocks_per_seq: int, mean_cache, num_slots: int, block: int, dtype: int,
                     params: Params) -> None:
    _check(lib().fp2_blockmean_cached(_ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                      _ptr(cu_seqlens), _ptr(block_table), max_blocks_per_seq,
                                      _ptr(mean_cache), num_slots, block, dtype,
                                      ctypes.byref(params)), "fp2_blockmean_cached")


def score(q, cu_seqlens, block: int, dtype: int, params: Params) -> None:
    _check(lib().fp2_score(_ptr(q), _ptr(cu_seqlens), block, dtype, ctypes.byref(params)),
           "fp2_score")


def mask(cu_seqlens, tau: float, block: int, params: Params) -> None:
    _check(lib().fp2_mask(_ptr(cu_seqlens), float(tau), block, ctypes.byref(params)), "fp2_mask")


def attn(q, k_cache, v_cache, page_table, cu_seqlens, kept_bits, block: int, dtype: int, out,
         params: Params) -> None:
    _check(lib().fp2_attn(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                          _ptr(cu_seqlens), _ptr(kept_bits), block, dtype, _ptr(out),
                          ctypes.byref(params)), "fp2_attn")


def workspace_init(params: Params) -> None:
    _check(lib().fp2_workspace_init(ctypes.byref(params)), "fp2_workspace_init")


def get_status(params: Params) -> tuple[int, int]:
    det = ctypes.c_uint32(0)
    st = lib().fp2_get_status(ctypes.byref(params), ctypes.byref(det))
    return int(st), int(det.value)


def noalloc_get_status(stream=None) -> tuple[int, int]:
    """Device-side status of the last fp2_prefill_noalloc call(s) on the
    current device; synchronises ``stream`` (default: torch's current one)."""
    if stream is None:
        import torch
        stream = torch.cuda.current_stream().cuda_stream
    det = ctypes.c_uint32(0)
    st = lib().fp2_noalloc_get_status(stream, ctypes.byref(det))
    return int(st), int(det.value)


def calibrate_tau(cu_seqlens, block: int, target_drop: float, params: Params) -> float:
    t = ctypes.c_float(0.0)
    _check(lib().fp2_calibrate_tau(_ptr(cu_seqlens), block, float(target_drop),
                                   ctypes.byref(params), ctypes.byref(t)), "fp2_calibrate_tau")
    return float(t.value)


# ---------------------------------------------------------------------------
# convenience: parameters from tensors, a torch-allocated workspace, views of
# the workspace's intermediates
# ---------------------------------------------------------------------------

@dataclass
class Problem:
    """Device tensors of one call plus its fp2_params (keeps them alive)."""
    q: object
    k: object
    v: object
    page_table: object
    cu_seqlens: object
    out: object
    block: int
    dtype: int
    params: Params
    workspace: object
    keep: tuple = ()

    def layout(self) -> WorkspaceLayout:
        return get_workspace_layout(self.params, self.block)

    def ws_view(self, name: str, torch_dtype, shape):
        """A tensor view of one workspace region (see WorkspaceLayout)."""
        import torch
        L = self.layout()
        off = getattr(L, name)
        n = 1
        for s in shape:
            n *= s
        itemsize = torch.empty((), dtype=torch_dtype).element_size()
        return self.workspace[off: off + n * itemsize].view(torch_dtype).view(*shape)

    def prefill(self, tau: float):
        prefill(self.q, self.k, self.v, self.page_table, self.cu_seqlens, tau, self.block,
                self.dtype, self.out, self.params)

    def check(self):
        st, det = get_status(self.params)
        if st != FP2_OK:
            raise Fp2Error(st, "device", det)


def make_problem(q, k, v, cu_seqlens, *, Hq: int, Hkv: int, d: int, block: int, dtype: int,
                 max_seqlen_q: int, max_seqlen_k: int, seqlens_k=None, cu_seqlens_k=None,
                 page_table=None, page_size: int = 0, q_scale=None, k_scale=None,
                 v_scale=None, out=None, stream=None, workspace=None,
                 group_masks: bool = False, out_dtype: int = FP2_BF16,
                 out_scale=None, attn_kernel: int = 0, k_block_factor=None,
                 v_block_factor=None) -> Problem:
    """Builds fp2_params for device tensors and allocates the workspace and
    the bf16 output with torch (allocation only)."""
    import torch
    dev = q.device
    P = Params()
    P.num_seqs = int(cu_seqlens.numel() - 1)
    P.num_q_heads, P.num_kv_heads, P.head_dim = Hq, Hkv, d
    P.total_q = int(q.shape[0])
    if page_table is None:
        P.total_k = int(k.shape[0])
    else:
        P.total_k = 0
        P.page_size = page_size
        P.max_pages_per_seq = int(page_table.shape[1])
        P.num_pages = int(k.shape[0])
    P.max_seqlen_q, P.max_seqlen_k = int(max_seqlen_q), int(max_seqlen_k)
    P.seqlens_k = _ptr(seqlens_k)
    P.cu_seqlens_k = _ptr(cu_seqlens_k)
    P.q_scale, P.k_scale, P.v_scale = _ptr(q_scale), _ptr(k_scale), _ptr(v_scale)
    P.group_masks = 1 if group_masks else 0
    P.out_dtype = out_dtype
    P.out_scale = _ptr(out_scale)
    P.attn_kernel = int(attn_kernel)
    P.k_block_factor = _ptr(k_block_factor)
    P.v_block_factor = _ptr(v_block_factor)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    P.stream = stream
    nbytes = workspace_size(P, block)
    if nbytes == 0:
        raise Fp2Error(FP2_ERR_INVALID_ARG, "fp2_workspace_size")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    P.workspace = workspace.data_ptr()
    P.workspace_bytes = workspace.numel()
    workspace_init(P)
    if out is None:
        odt = torch.float8_e4m3fn if out_dtype == FP2_FP8_E4M3 else torch.bfloat16
        out = torch.empty((q.shape[0], Hq, d), dtype=odt, device=dev)
    keep = (seqlens_k, cu_seqlens_k, q_scale, k_scale, v_scale, out_scale, k_block_factor,
            v_block_factor)
    return Problem(q, k, v, page_table, cu_seqlens, out, block, dtype, P, workspace, keep)
