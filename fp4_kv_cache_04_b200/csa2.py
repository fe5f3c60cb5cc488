"""Python binding of libcsa2.so (ctypes).  Argument marshalling only: every step of the
CSA2 path runs in the library's CUDA kernels.  Tensors are torch CUDA tensors (torch is
used for device memory and streams); each function has the name of its C entry point
without the ``csa2_`` prefix.  Errors raise ``Csa2Error`` with the library's status.

There is no fallback: if the shared library is missing or fails to load, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libcsa2.so not built at {LIB_PATH}; run __graft_entry__.build() "
                      "or python -m fp4_kv_cache_04_b200.build")
_lib = ctypes.CDLL(LIB_PATH)

# Constants mirrored from include/csa2.h
D = 512
GROUP = 16
ROW_CODES = 256
ROW_SCALES = 32
HEADS = 16
IDX_HEADS = 4
IDX_DIM = 64
TOPK = 512
WINDOW = 128
POOL_BLOCKS = 2048
POOL_BLOCK = 8
MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2
CACHE_OFF, CACHE_FILL, CACHE_USE = 0, 1, 2
SWA_BF16, SWA_FP8 = 0, 1
Q_BF16, Q_NVFP4 = 0, 1

OK = 0
STATUS_NAMES = {0: "CSA2_OK", 1: "CSA2_ERR_INVALID_ARG", 2: "CSA2_ERR_UNSUPPORTED",
                3: "CSA2_ERR_WORKSPACE", 4: "CSA2_ERR_CUDA", 5: "CSA2_ERR_TIMEOUT",
                6: "CSA2_ERR_DEVICE"}

EXPORTED = ["csa2_status_string", "csa2_last_error", "csa2_abi_version",
            "csa2_kernel_launches", "csa2_quantize_kv", "csa2_append_kv",
            "csa2_index_score", "csa2_topk", "csa2_pool_workspace_size", "csa2_build_pool",
            "csa2_build_pool_noalloc",
            "csa2_workspace_size", "csa2_attend", "csa2_check_device_status", "csa2_set_wait_limit"]


class Csa2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = _lib.csa2_last_error().decode() if status == 4 else ""
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} {detail}".strip())


class IndexArgs(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("q_per_seq", ctypes.c_int32),
                ("ratio", ctypes.c_int32), ("reserved0", ctypes.c_int32),
                ("max_n", ctypes.c_int64), ("kv_offsets", ctypes.c_void_p),
                ("q_pos", ctypes.c_void_p), ("idx_q", ctypes.c_void_p),
                ("idx_w", ctypes.c_void_p), ("idx_k", ctypes.c_void_p),
                ("idx_kscale", ctypes.c_void_p), ("pool_blocks", ctypes.c_void_p)]


class LayerArgs(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("q_per_seq", ctypes.c_int32), ("ratio", ctypes.c_int32),
                ("want_pool", ctypes.c_int32), ("reserved0", ctypes.c_int32),
                ("max_n", ctypes.c_int64), ("total_n", ctypes.c_int64),
                ("kv_offsets", ctypes.c_void_p), ("q_pos", ctypes.c_void_p),
                ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("idx_q", ctypes.c_void_p),
                ("idx_w", ctypes.c_void_p), ("idx_k", ctypes.c_void_p),
                ("idx_kscale", ctypes.c_void_p), ("pool_blocks", ctypes.c_void_p),
                ("topk_idx", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("swa_kv", ctypes.c_void_p), ("swa_rows", ctypes.c_int64),
                ("sm_scale", ctypes.c_float), ("reserved1", ctypes.c_int32),
                ("out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("sel_cache", ctypes.c_void_p),
                ("sel_cache_mode", ctypes.c_int32), ("swa_format", ctypes.c_int32),
                ("ev_index_begin", ctypes.c_void_p), ("ev_index_end", ctypes.c_void_p),
                ("swa_kv8", ctypes.c_void_p), ("swa_kscale", ctypes.c_void_p),
                ("pool_k", ctypes.c_void_p), ("pool_kscale", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("page_rows", ctypes.c_int32),
                ("pages_per_seq", ctypes.c_int32), ("q_format", ctypes.c_int32),
                ("reserved2", ctypes.c_int32), ("ev_pool", ctypes.c_void_p)]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_lib.csa2_status_string.restype = ctypes.c_char_p
_lib.csa2_status_string.argtypes = [_i32]
_lib.csa2_last_error.restype = ctypes.c_char_p
_lib.csa2_abi_version.restype = _i32
_lib.csa2_kernel_launches.restype = ctypes.c_uint64
_lib.csa2_quantize_kv.restype = _i32
_lib.csa2_quantize_kv.argtypes = [_vp, _i64, _i32, _vp, _vp, _vp, _vp]
_lib.csa2_append_kv.restype = _i32
_lib.csa2_append_kv.argtypes = [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.csa2_index_score.restype = _i32
_lib.csa2_index_score.argtypes = [ctypes.POINTER(IndexArgs), _vp, _i64, _vp]
_lib.csa2_topk.restype = _i32
_lib.csa2_topk.argtypes = [_vp, _i64, _i64, _i32, _i32, _vp, _i32, _vp, _vp]
_lib.csa2_pool_workspace_size.restype = _sz
_lib.csa2_pool_workspace_size.argtypes = [_i32, _i64]
_lib.csa2_build_pool.restype = _i32
_lib.csa2_build_pool.argtypes = [_vp, _i64, _vp, _i32, _i64, _vp, _vp, _sz, _vp]
_lib.csa2_build_pool_noalloc.restype = _i32
_lib.csa2_build_pool_noalloc.argtypes = [_vp, _i64, _vp, _i32, _i64, _vp, _vp]
_lib.csa2_workspace_size.restype = _sz
_lib.csa2_workspace_size.argtypes = [ctypes.POINTER(LayerArgs)]
_lib.csa2_attend.restype = _i32
_lib.csa2_attend.argtypes = [ctypes.POINTER(LayerArgs), _vp]
_lib.csa2_check_device_status.restype = _i32
_lib.csa2_check_device_status.argtypes = [_vp, _vp]
_lib.csa2_set_wait_limit.restype = _i32
_lib.csa2_set_wait_limit.argtypes = [_vp, ctypes.c_uint32, _vp]


def lib() -> ctypes.CDLL:
    return _lib


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libcsa2 takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libcsa2 takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str) -> None:
    if status != OK:
        raise Csa2Error(status, where)


def abi_version() -> int:
    return _lib.csa2_abi_version()


def kernel_launches() -> int:
    return _lib.csa2_kernel_launches()


def status_string(status: int) -> str:
    return _lib.csa2_status_string(status).decode()


def quantize_kv(x: torch.Tensor, ratio: int, codes: torch.Tensor, scales: torch.Tensor,
                dst_row: torch.Tensor | None = None, stream=None) -> None:
    """bf16 rows [n][512] -> codes [rows][256] u8 + scales [rows][32] u8 (see csa2.h)."""
    assert x.dtype == torch.bfloat16 and codes.dtype == torch.uint8 and scales.dtype == torch.uint8
    _check(_lib.csa2_quantize_kv(_ptr(x), x.shape[0] if x.dim() else 0, ratio, _ptr(dst_row),
                                 _ptr(codes), _ptr(scales), _stream(stream)), "csa2_quantize_kv")


def append_kv(latent: torch.Tensor, idx_proj: torch.Tensor, dst_row: torch.Tensor, codes: torch.Tensor,
              scales: torch.Tensor, idx_k: torch.Tensor, idx_kscale: torch.Tensor, stream=None) -> None:
    """New decode positions: bf16 latent [n][512] and fp32 indexer values [n][64] ->
    FP4 main-KV rows and FP8 indexer-K rows (+ fp32 scales) at rows dst_row."""
    _check(_lib.csa2_append_kv(_ptr(latent), _ptr(idx_proj), latent.shape[0], _ptr(dst_row), _ptr(codes),
                               _ptr(scales), _ptr(idx_k), _ptr(idx_kscale), _stream(stream)), "csa2_append_kv")


def _index_args(batch, q_per_seq, ratio, max_n, kv_offsets, q_pos, idx_q, idx_w, idx_k,
                idx_kscale, pool_blocks) -> IndexArgs:
    return IndexArgs(batch, q_per_seq, ratio, 0, max_n, _ptr(kv_offsets), _ptr(q_pos),
                     _ptr(idx_q), _ptr(idx_w), _ptr(idx_k), _ptr(idx_kscale), _ptr(pool_blocks))


def index_score(*, batch, q_per_seq, max_n, kv_offsets, idx_q, idx_w, idx_k, idx_kscale,
                scores, ratio=1, q_pos=None, pool_blocks=None, stream=None) -> None:
    a = _index_args(batch, q_per_seq, ratio, max_n, kv_offsets, q_pos, idx_q, idx_w, idx_k,
                    idx_kscale, pool_blocks)
    _check(_lib.csa2_index_score(ctypes.byref(a), _ptr(scores), scores.stride(0), _stream(stream)),
           "csa2_index_score")


def topk(scores: torch.Tensor, n_cols: int, k: int, idx_out: torch.Tensor,
         pool_blocks: torch.Tensor | None = None, q_per_seq: int = 1, stream=None) -> None:
    _check(_lib.csa2_topk(_ptr(scores), scores.stride(0), n_cols, scores.shape[0], k,
                          _ptr(pool_blocks), q_per_seq, _ptr(idx_out), _stream(stream)),
           "csa2_topk")


def pool_workspace_size(batch: int, max_n: int) -> int:
    return _lib.csa2_pool_workspace_size(batch, max_n)


def build_pool(scores: torch.Tensor, kv_offsets: torch.Tensor, max_n: int,
               pool_blocks: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _check(_lib.csa2_build_pool(_ptr(scores), scores.stride(0), _ptr(kv_offsets), scores.shape[0],
                                max_n, _ptr(pool_blocks), _ptr(workspace), workspace.numel(),
                                _stream(stream)), "csa2_build_pool")


NOALLOC_POOL_SCRATCH_BYTES = 8 << 20


def build_pool_noalloc(scores: torch.Tensor, kv_offsets: torch.Tensor, max_n: int,
                       pool_blocks: torch.Tensor, stream=None) -> None:
    _check(_lib.csa2_build_pool_noalloc(_ptr(scores), scores.stride(0), _ptr(kv_offsets),
                                        scores.shape[0], max_n, _ptr(pool_blocks),
                                        _stream(stream)), "csa2_build_pool_noalloc")


def layer_args(*, mode, batch, q_per_seq, max_n, kv_offsets, codes, scales, topk_idx, q, swa_kv,
               out, workspace=None, ratio=1, want_pool=False, q_pos=None, idx_q=None, idx_w=None,
               idx_k=None, idx_kscale=None, pool_blocks=None, swa_rows=None, sm_scale=1.0,
               ev_index_begin=None, ev_index_end=None, total_n=None, sel_cache=None,
               sel_cache_mode=0, swa_kv8=None, swa_kscale=None, pool_k=None, pool_kscale=None,
               page_table=None, page_rows=0, q_nvfp4=False, ev_pool=None) -> LayerArgs:
    """swa_kv: bf16 [B][rows][512]; or pass swa_kv=None with swa_kv8 (E4M3 [B][rows][512])
    and swa_kscale (fp32 [B][rows]) for the FP8 SWA format.  pool_k (uint8 [B][16384][64])
    and pool_kscale (fp32 [B][16384]): the HSI pool's rows, contiguous (written by a FULL
    call with want_pool, streamed by REINDEX calls).  page_table (int32 [B][pages]) with
    page_rows: a paged cache (row of position p of sequence b = page_table[b][p // page_rows]
    * page_rows + p % page_rows).  q_nvfp4: the block-scaled FP4 query variant
    (CSA2_Q_NVFP4).  ev_pool (torch.cuda.Event): a FULL call with want_pool records it
    instead of joining its pool work into the stream; a REINDEX call waits for it."""
    swa_format = SWA_FP8 if swa_kv8 is not None else SWA_BF16
    if swa_rows is None:
        swa_rows = (swa_kv8 if swa_kv8 is not None else swa_kv).shape[1]
    if total_n is None:
        total_n = codes.shape[0]           # rows of the packed caches
    return LayerArgs(mode, batch, q_per_seq, ratio, int(bool(want_pool)), 0, max_n, total_n,
                     _ptr(kv_offsets), _ptr(q_pos), _ptr(codes), _ptr(scales), _ptr(idx_q),
                     _ptr(idx_w), _ptr(idx_k), _ptr(idx_kscale), _ptr(pool_blocks),
                     _ptr(topk_idx), _ptr(q), _ptr(swa_kv), swa_rows, sm_scale, 0, _ptr(out),
                     _ptr(workspace), workspace.numel() if workspace is not None else 0,
                     _ptr(sel_cache), sel_cache_mode, swa_format, _event(ev_index_begin),
                     _event(ev_index_end), _ptr(swa_kv8), _ptr(swa_kscale), _ptr(pool_k), _ptr(pool_kscale),
                     _ptr(page_table), int(page_rows), 0 if page_table is None else page_table.shape[1],
                     Q_NVFP4 if q_nvfp4 else Q_BF16, 0, _event(ev_pool))


def _event(ev) -> int | None:
    """torch.cuda.Event -> its cudaEvent_t handle (the event is created if needed)."""
    if ev is None:
        return None
    if isinstance(ev, int):
        return ev
    if ev.cuda_event == 0:
        ev.record()                      # torch creates the CUDA event lazily
        torch.cuda.current_stream().synchronize()
    return ev.cuda_event


def workspace_size(args: LayerArgs) -> int:
    return _lib.csa2_workspace_size(ctypes.byref(args))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zeroed workspace (the device error word starts cleared)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def attend(args: LayerArgs, stream=None) -> None:
    _check(_lib.csa2_attend(ctypes.byref(args), _stream(stream)), "csa2_attend")


def attend_status(args: LayerArgs, stream=None) -> int:
    """csa2_attend returning the raw status instead of raising (for validation tests)."""
    return _lib.csa2_attend(ctypes.byref(args), _stream(stream))


def check_device_status(workspace: torch.Tensor, stream=None) -> int:
    return _lib.csa2_check_device_status(_ptr(workspace), _stream(stream))


def set_wait_limit(workspace: torch.Tensor, polls: int, stream=None) -> None:
    """Bound (in polls) of the device-side waits of later calls with this workspace; 0 =
    the library default."""
    _check(_lib.csa2_set_wait_limit(_ptr(workspace), int(polls), _stream(stream)), "csa2_set_wait_limit")
