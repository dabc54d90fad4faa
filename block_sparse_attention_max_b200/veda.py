"""ctypes binding of libveda.so (include/veda.h) -- argument marshalling only.

Every step of the path runs in the library's CUDA kernels; this module only turns
torch tensors into pointers and sizes, allocates outputs with torch, and raises when
a call returns an error. There is no fallback: if the library is missing or the device
is not a B200 (compute capability 10.0), calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libveda.so")

VEDA_OK = 0
STATUS_NAMES = {0: "VEDA_OK", 1: "VEDA_ERR_INVALID_ARG", 2: "VEDA_ERR_UNSUPPORTED",
                3: "VEDA_ERR_CUDA", 4: "VEDA_ERR_TIMEOUT", 5: "VEDA_ERR_DEVICE_CHECK"}

EXPORTED = (
    "veda_abi_version", "veda_status_string", "veda_last_error", "veda_geometry_sizes",
    "veda_build_tile_map", "veda_permute_tiles", "veda_permute_pool", "veda_tile_pool",
    "veda_block_scores_workspace_bytes", "veda_block_scores", "veda_block_scores_noalloc",
    "veda_select_blocks",
    "veda_block_sparse_attn_fwd", "veda_unpermute", "veda_transpose_lists",
    "veda_block_sparse_attn_bwd", "veda_block_heat", "veda_mask_quality", "veda_rel_error",
    "veda_tile_plan_vote",
    "veda_quantize_fp8", "veda_block_sparse_attn_fwd_fp8",
    "veda_check_device_status", "veda_selftest_wait_timeout",
)


class VedaError(RuntimeError):
    def __init__(self, call: str, status: int, message: str):
        super().__init__(f"{call} -> {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class TileShape(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int32), ("h", ctypes.c_int32), ("w", ctypes.c_int32)]


class Geometry(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("T", ctypes.c_int32), ("Hg", ctypes.c_int32),
                ("Wg", ctypes.c_int32), ("n_tail", ctypes.c_int32),
                ("head_shape", ctypes.POINTER(TileShape)),
                ("tile_order", ctypes.POINTER(ctypes.c_int32)),
                ("order_stride", ctypes.c_int32)]


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SIG = {
    "veda_abi_version": (_I, []),
    "veda_status_string": (ctypes.c_char_p, [_I]),
    "veda_last_error": (ctypes.c_char_p, []),
    "veda_geometry_sizes": (_I, [ctypes.POINTER(Geometry), _P, _P, _P]),
    "veda_build_tile_map": (_I, [ctypes.POINTER(Geometry), _P, _P, _P, _P]),
    "veda_permute_tiles": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "veda_tile_pool": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "veda_permute_pool": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "veda_block_scores_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "veda_block_scores": (_I, [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _P]),
    "veda_block_scores_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "veda_select_blocks": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "veda_block_sparse_attn_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _F, _P, _P, _I, _I,
                                        _I, _I, _P]),
    "veda_unpermute": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "veda_quantize_fp8": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "veda_block_sparse_attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _F, _P, _P,
                                            _I, _I, _I, _I, _P]),
    "veda_transpose_lists": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P]),
    "veda_block_sparse_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I,
                                        _F, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "veda_rel_error": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "veda_tile_plan_vote": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "veda_block_heat": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _F, _P, _I, _I, _I, _I, _P]),
    "veda_mask_quality": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I, _P, _P, _P,
                               _I, _I, _I, _P]),
    "veda_check_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "veda_selftest_wait_timeout": (_I, [ctypes.c_uint32, _P]),
}


def lib() -> ctypes.CDLL:
    """The loaded library. Raises if libveda.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_attention_max_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIG.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(call: str, status: int) -> None:
    if status != VEDA_OK:
        msg = lib().veda_last_error().decode(errors="replace")
        raise VedaError(call, status, msg)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, cuda: bool = True,
          shape: Optional[Sequence[int]] = None) -> None:
    """Type, shape, layout and device of a tensor handed to the library: a wrong shape would
    send a kernel outside the buffer, so every one is checked before its pointer is passed."""
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name}: expected shape {tuple(int(x) for x in shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if cuda and t.device.index != torch.cuda.current_device():
        # the library launches on the calling thread's current device
        raise ValueError(f"{name}: on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")


def _need_maps(maps: "DeviceMaps", H: int, Npad: int, cuda: bool = True) -> None:
    """The device tile map of H heads with Npad slots each (and its per-tile arrays)."""
    if maps.Npad != Npad or maps.nT * 128 != Npad:
        raise ValueError(f"tile map of {maps.Npad} slots per head, tensors have {Npad}")
    _need(maps.tile_map, torch.int32, "tile_map", cuda, shape=(H, Npad))
    for t, n in ((maps.tile_valid, "tile_valid"), (maps.tile_segment, "tile_segment")):
        _need(t, torch.int32, n, cuda, shape=(H, Npad // 128))
    _need(maps.nT_per_head, torch.int32, "nT_per_head", cuda, shape=(H,))


def _need_lists(lists: "BlockLists", B: int, H: int, nT: int, name: str = "lists", cuda: bool = True) -> None:
    """Block lists of a [B, H, nT] problem: counts [B, H, nT], indices [B, H, nT, stride]."""
    if not 0 < lists.stride <= nT:
        raise ValueError(f"{name}: stride {lists.stride} outside [1, {nT}]")
    for t, n in ((lists.full_cnt, "full_cnt"), (lists.part_cnt, "part_cnt")):
        _need(t, torch.int32, f"{name}.{n}", cuda, shape=(B, H, nT))
    for t, n in ((lists.full_idx, "full_idx"), (lists.part_idx, "part_idx")):
        _need(t, torch.int32, f"{name}.{n}", cuda, shape=(B, H, nT, lists.stride))


# ---------------------------------------------------------------------------------------
# geometry (host)
# ---------------------------------------------------------------------------------------

@dataclasses.dataclass
class TileMaps:
    """Host tile maps of one geometry (numpy int32)."""
    tile_map: np.ndarray       # [H, Npad]
    tile_valid: np.ndarray     # [H, nT]
    tile_segment: np.ndarray   # [H, nT]
    nT_per_head: np.ndarray    # [H]
    N: int
    nT: int
    Npad: int

    def to(self, device) -> "DeviceMaps":
        f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        return DeviceMaps(f(self.tile_map), f(self.tile_valid), f(self.tile_segment),
                          f(self.nT_per_head), self.N, self.nT, self.Npad)


@dataclasses.dataclass
class DeviceMaps:
    tile_map: torch.Tensor
    tile_valid: torch.Tensor
    tile_segment: torch.Tensor
    nT_per_head: torch.Tensor
    N: int
    nT: int
    Npad: int


def _geometry(grid, head_shapes, n_tail, tile_order):
    H = len(head_shapes)
    shapes = (TileShape * H)(*[TileShape(*map(int, s)) for s in head_shapes])
    keep = [shapes]
    g = Geometry(H, int(grid[0]), int(grid[1]), int(grid[2]), int(n_tail), shapes, None, 0)
    if tile_order is not None:
        order = np.ascontiguousarray(np.asarray(tile_order, dtype=np.int32))
        keep.append(order)
        g.tile_order = order.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        g.order_stride = order.shape[1]
    return g, keep


def geometry_sizes(grid, head_shapes, n_tail=0) -> Tuple[int, int, int]:
    g, _keep = _geometry(grid, head_shapes, n_tail, None)
    N, nT, Npad = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check("veda_geometry_sizes", lib().veda_geometry_sizes(
        ctypes.byref(g), ctypes.addressof(N), ctypes.addressof(nT), ctypes.addressof(Npad)))
    return N.value, nT.value, Npad.value


def build_tile_map(grid, head_shapes, n_tail=0, tile_order=None) -> TileMaps:
    g, _keep = _geometry(grid, head_shapes, n_tail, tile_order)
    N, nT, Npad = geometry_sizes(grid, head_shapes, n_tail)
    H = len(head_shapes)
    tm = np.empty((H, Npad), np.int32)
    tv = np.empty((H, nT), np.int32)
    ts = np.empty((H, nT), np.int32)
    nph = np.empty((H,), np.int32)
    _check("veda_build_tile_map", lib().veda_build_tile_map(
        ctypes.byref(g), tm.ctypes.data, tv.ctypes.data, ts.ctypes.data, nph.ctypes.data))
    return TileMaps(tm, tv, ts, nph, N, nT, Npad)


# ---------------------------------------------------------------------------------------
# device steps
# ---------------------------------------------------------------------------------------

def permute_tiles(x: torch.Tensor, maps: DeviceMaps, out: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    _need(x, torch.bfloat16, "x")
    B, N, H, D = x.shape
    _need_maps(maps, H, maps.Npad)
    if out is None:
        out = torch.empty((B, H, maps.Npad, D), dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, "out", shape=(B, H, maps.Npad, D))
    _check("veda_permute_tiles", lib().veda_permute_tiles(
        _ptr(x), _ptr(out), _ptr(maps.tile_map), B, N, H, D, maps.Npad, _stream(stream)))
    return out


def permute_pool(x: torch.Tensor, maps: DeviceMaps, out: Optional[torch.Tensor] = None,
                 pooled: Optional[torch.Tensor] = None, stream=None):
    """veda_permute_pool: the tile gather and the tile pooling in one pass."""
    _need(x, torch.bfloat16, "x")
    B, N, H, D = x.shape
    _need_maps(maps, H, maps.Npad)
    if out is None:
        out = torch.empty((B, H, maps.Npad, D), dtype=torch.bfloat16, device=x.device)
    if pooled is None:
        pooled = torch.empty((B, H, maps.Npad // 128, 3, D), dtype=torch.float32, device=x.device)
    _need(out, torch.bfloat16, "out", shape=(B, H, maps.Npad, D))
    _need(pooled, torch.float32, "pooled", shape=(B, H, maps.Npad // 128, 3, D))
    _check("veda_permute_pool", lib().veda_permute_pool(
        _ptr(x), _ptr(out), _ptr(maps.tile_map), _ptr(maps.tile_valid), _ptr(pooled), B, N, H, D,
        maps.Npad, _stream(stream)))
    return out, pooled


def tile_pool(x_tiled: torch.Tensor, maps: DeviceMaps, out: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    _need(x_tiled, torch.bfloat16, "x_tiled")
    B, H, Npad, D = x_tiled.shape
    nT = Npad // 128
    _need_maps(maps, H, Npad)
    if out is None:
        out = torch.empty((B, H, nT, 3, D), dtype=torch.float32, device=x_tiled.device)
    _need(out, torch.float32, "out", shape=(B, H, nT, 3, D))
    _check("veda_tile_pool", lib().veda_tile_pool(
        _ptr(x_tiled), _ptr(maps.tile_valid), _ptr(out), B, H, nT, D, _stream(stream)))
    return out


def block_scores_workspace_bytes(B: int, H: int, nT: int, D: int = 128) -> int:
    return int(lib().veda_block_scores_workspace_bytes(B, H, nT, D))


def block_scores(pooled_q: torch.Tensor, pooled_k: torch.Tensor, wq: torch.Tensor,
                 wk: torch.Tensor, out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need(pooled_q, torch.float32, "pooled_q")
    B, H, nT, three, D = pooled_q.shape
    if three != 3:
        raise ValueError("pooled_q: expected shape [B, H, nT, 3, D]")
    _need(pooled_k, torch.float32, "pooled_k", shape=pooled_q.shape)
    for t, n in ((wq, "wq"), (wk, "wk")):
        _need(t, torch.float32, n, shape=(H, D, 3 * D))
    if out is None:
        out = torch.empty((B, H, nT, nT), dtype=torch.float32, device=pooled_q.device)
    _need(out, torch.float32, "out", shape=(B, H, nT, nT))
    nbytes = block_scores_workspace_bytes(B, H, nT, D)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=pooled_q.device)
    _need(workspace, workspace.dtype, "workspace")
    _check("veda_block_scores", lib().veda_block_scores(
        _ptr(pooled_q), _ptr(pooled_k), _ptr(wq), _ptr(wk), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, H, nT, D, _stream(stream)))
    return out


def block_scores_noalloc(pooled_q: torch.Tensor, pooled_k: torch.Tensor, wq: torch.Tensor,
                         wk: torch.Tensor, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """veda_block_scores_noalloc: same result as block_scores, scratch built into the library.

    For callers that may not allocate device memory (see include/veda.h); ``out`` should
    then be passed in. Calls sharing a device must not overlap on the GPU.
    """
    for t, n in ((pooled_q, "pooled_q"), (pooled_k, "pooled_k"), (wq, "wq"), (wk, "wk")):
        _need(t, torch.float32, n)
    B, H, nT, three, D = pooled_q.shape
    if three != 3 or tuple(pooled_k.shape) != tuple(pooled_q.shape):
        raise ValueError("pooled_q / pooled_k: expected equal shapes [B, H, nT, 3, D]")
    for t, n in ((wq, "wq"), (wk, "wk")):
        if tuple(t.shape) != (H, D, 3 * D):
            raise ValueError(f"{n}: expected shape {(H, D, 3 * D)}, got {tuple(t.shape)}")
    if out is None:
        out = torch.empty((B, H, nT, nT), dtype=torch.float32, device=pooled_q.device)
    _need(out, torch.float32, "out")
    if tuple(out.shape) != (B, H, nT, nT):
        raise ValueError(f"out: expected shape {(B, H, nT, nT)}, got {tuple(out.shape)}")
    _check("veda_block_scores_noalloc", lib().veda_block_scores_noalloc(
        _ptr(pooled_q), _ptr(pooled_k), _ptr(wq), _ptr(wk), _ptr(out), B, H, nT, D,
        _stream(stream)))
    return out


def list_stride_for(nT: int, rho: Sequence[Tuple[int, int]]) -> int:
    """Smallest list_stride veda_select_blocks accepts for these densities."""
    bound = 1 + sum(-(-nT * p // q) for p, q in rho)
    return min(nT, bound)


@dataclasses.dataclass
class BlockLists:
    full_cnt: torch.Tensor    # [B, H, nT] int32
    full_idx: torch.Tensor    # [B, H, nT, stride] int32
    part_cnt: torch.Tensor
    part_idx: torch.Tensor
    stride: int


def select_blocks(scores: torch.Tensor, maps: DeviceMaps, rho: Sequence[Tuple[int, int]],
                  list_stride: Optional[int] = None, out: Optional[BlockLists] = None,
                  stream=None) -> BlockLists:
    _need(scores, torch.float32, "scores")
    B, H, nT, nT2 = scores.shape
    if nT2 != nT:
        raise ValueError("scores: expected shape [B, H, nT, nT]")
    _need_maps(maps, H, nT * 128)
    stride = list_stride or list_stride_for(nT, rho)
    if out is None:
        dev = scores.device
        out = BlockLists(torch.empty((B, H, nT), dtype=torch.int32, device=dev),
                         torch.zeros((B, H, nT, stride), dtype=torch.int32, device=dev),
                         torch.empty((B, H, nT), dtype=torch.int32, device=dev),
                         torch.zeros((B, H, nT, stride), dtype=torch.int32, device=dev), stride)
    _need_lists(out, B, H, nT, "out")
    num = (ctypes.c_int32 * len(rho))(*[int(p) for p, _ in rho])
    den = (ctypes.c_int32 * len(rho))(*[int(q) for _, q in rho])
    _check("veda_select_blocks", lib().veda_select_blocks(
        _ptr(scores), _ptr(maps.tile_valid), _ptr(maps.tile_segment), _ptr(maps.nT_per_head),
        len(rho), ctypes.addressof(num), ctypes.addressof(den), _ptr(out.full_cnt),
        _ptr(out.full_idx), _ptr(out.part_cnt), _ptr(out.part_idx), out.stride, B, H, nT,
        _stream(stream)))
    return out


def block_sparse_attn_fwd(q_t: torch.Tensor, k_t: torch.Tensor, v_t: torch.Tensor,
                          maps: DeviceMaps, lists: BlockLists, scale: float,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                          want_lse: bool = True, stream=None):
    _need(q_t, torch.bfloat16, "q")
    B, H, Npad, D = q_t.shape
    nT = Npad // 128
    for t, n in ((k_t, "k"), (v_t, "v")):
        _need(t, torch.bfloat16, n, shape=q_t.shape)
    _need_maps(maps, H, Npad)
    _need_lists(lists, B, H, nT)
    if out is None:
        out = torch.empty_like(q_t)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q_t.device)
    _need(out, torch.bfloat16, "out", shape=q_t.shape)
    if lse is not None:
        _need(lse, torch.float32, "lse", shape=(B, H, Npad))
    _check("veda_block_sparse_attn_fwd", lib().veda_block_sparse_attn_fwd(
        _ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(maps.tile_valid), _ptr(lists.full_cnt),
        _ptr(lists.full_idx), _ptr(lists.part_cnt), _ptr(lists.part_idx), lists.stride,
        float(scale), _ptr(out), _ptr(lse), B, H, nT, D, _stream(stream)))
    return out, lse


def quantize_fp8(x_t: torch.Tensor, transpose_tiles: bool = False, codes: Optional[torch.Tensor] = None,
                 scale: Optional[torch.Tensor] = None, stream=None):
    """Tiled bf16 [B, H, Npad, 128] -> (e4m3 codes uint8 [B, H, Npad, 128], scale fp32 [B, H]);
    with transpose_tiles every 128 x 128 tile of the codes is stored transposed, keys in the
    order veda_quantize_fp8 documents (V of the FP8 attention)."""
    _need(x_t, torch.bfloat16, "x_t")
    B, H, Npad, D = x_t.shape
    if codes is None:
        codes = torch.empty((B, H, Npad, D), dtype=torch.uint8, device=x_t.device)
    if scale is None:
        scale = torch.empty((B, H), dtype=torch.float32, device=x_t.device)
    _need(codes, torch.uint8, "codes", shape=(B, H, Npad, D))
    _need(scale, torch.float32, "scale", shape=(B, H))
    _check("veda_quantize_fp8", lib().veda_quantize_fp8(
        _ptr(x_t), _ptr(codes), _ptr(scale), B, H, Npad // 128, D, 1 if transpose_tiles else 0, _stream(stream)))
    return codes, scale


def block_sparse_attn_fwd_fp8(q8: torch.Tensor, k8: torch.Tensor, vt8: torch.Tensor, q_scale: torch.Tensor,
                              k_scale: torch.Tensor, v_scale: torch.Tensor, maps: DeviceMaps, lists: BlockLists,
                              scale: float, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                              want_lse: bool = True, stream=None):
    """FP8 variant of the attention step: e4m3 codes of Q, K and (transposed tiles) V with
    their per-(batch, head) scales -> bf16 O [B, H, Npad, 128] and fp32 LSE."""
    _need(q8, torch.uint8, "q8")
    B, H, Npad, D = q8.shape
    nT = Npad // 128
    for t, n in ((k8, "k8"), (vt8, "vt8")):
        _need(t, torch.uint8, n, shape=q8.shape)
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, torch.float32, n, shape=(B, H))
    _need_maps(maps, H, Npad)
    _need_lists(lists, B, H, nT)
    if out is None:
        out = torch.empty((B, H, Npad, D), dtype=torch.bfloat16, device=q8.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q8.device)
    _need(out, torch.bfloat16, "out", shape=(B, H, Npad, D))
    if lse is not None:
        _need(lse, torch.float32, "lse", shape=(B, H, Npad))
    _check("veda_block_sparse_attn_fwd_fp8", lib().veda_block_sparse_attn_fwd_fp8(
        _ptr(q8), _ptr(k8), _ptr(vt8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _ptr(maps.tile_valid),
        _ptr(lists.full_cnt), _ptr(lists.full_idx), _ptr(lists.part_cnt), _ptr(lists.part_idx), lists.stride,
        float(scale), _ptr(out), _ptr(lse), B, H, nT, D, _stream(stream)))
    return out, lse


@dataclasses.dataclass
class TransposedLists:
    cnt: torch.Tensor    # [B, H, nT] int32: query tiles per key tile
    idx: torch.Tensor    # [B, H, nT, stride] int32, ascending
    stride: int


def transpose_lists(lists: BlockLists, maps: DeviceMaps, stream=None) -> TransposedLists:
    """veda_transpose_lists: the query tiles of every key tile (the backward's lists)."""
    B, H, nT = lists.full_cnt.shape
    _need_lists(lists, B, H, nT)
    _need_maps(maps, H, nT * 128)
    dev = lists.full_cnt.device
    t = TransposedLists(torch.empty((B, H, nT), dtype=torch.int32, device=dev),
                        torch.zeros((B, H, nT, nT), dtype=torch.int32, device=dev), nT)
    _check("veda_transpose_lists", lib().veda_transpose_lists(
        _ptr(lists.full_cnt), _ptr(lists.full_idx), _ptr(lists.part_cnt), _ptr(lists.part_idx),
        lists.stride, _ptr(maps.nT_per_head), _ptr(t.cnt), _ptr(t.idx), t.stride, B, H, nT,
        _stream(stream)))
    return t


def block_sparse_attn_bwd(q_t: torch.Tensor, k_t: torch.Tensor, v_t: torch.Tensor, o_t: torch.Tensor,
                          do_t: torch.Tensor, lse: torch.Tensor, maps: DeviceMaps, lists: BlockLists,
                          tlists: TransposedLists, scale: float, stream=None):
    """veda_block_sparse_attn_bwd: dQ, dK, dV (tile order, bf16) over the forward's lists."""
    _need(q_t, torch.bfloat16, "q")
    B, H, Npad, D = q_t.shape
    nT = Npad // 128
    for t, n in ((k_t, "k"), (v_t, "v"), (o_t, "o"), (do_t, "dout")):
        _need(t, torch.bfloat16, n, shape=q_t.shape)
    _need(lse, torch.float32, "lse", shape=(B, H, Npad))
    _need_maps(maps, H, Npad)
    _need_lists(lists, B, H, nT)
    if tlists.stride != nT:
        raise ValueError(f"tlists: stride {tlists.stride}, expected {nT}")
    _need(tlists.cnt, torch.int32, "tlists.cnt", shape=(B, H, nT))
    _need(tlists.idx, torch.int32, "tlists.idx", shape=(B, H, nT, nT))
    dq, dk, dv = torch.empty_like(q_t), torch.empty_like(k_t), torch.empty_like(v_t)
    delta = torch.empty(B * H * Npad + 4, dtype=torch.float32, device=q_t.device)   # D + work counters
    _check("veda_block_sparse_attn_bwd", lib().veda_block_sparse_attn_bwd(
        _ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(o_t), _ptr(do_t), _ptr(lse), _ptr(maps.tile_valid),
        _ptr(lists.full_cnt), _ptr(lists.full_idx), _ptr(lists.part_cnt), _ptr(lists.part_idx),
        lists.stride, _ptr(tlists.cnt), _ptr(tlists.idx), tlists.stride, float(scale), _ptr(dq),
        _ptr(dk), _ptr(dv), _ptr(delta), B, H, nT, D, _stream(stream)))
    return dq, dk, dv


def block_heat(q_t: torch.Tensor, k_t: torch.Tensor, maps: DeviceMaps, lists: BlockLists,
               lse: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """veda_block_heat: per-block attention mass against the given (dense) LSE."""
    _need(q_t, torch.bfloat16, "q")
    B, H, Npad, D = q_t.shape
    nT = Npad // 128
    _need(k_t, torch.bfloat16, "k", shape=q_t.shape)
    _need(lse, torch.float32, "lse", shape=(B, H, Npad))
    _need_maps(maps, H, Npad)
    _need_lists(lists, B, H, nT)
    if out is None:
        out = torch.empty((B, H, nT, nT), dtype=torch.float32, device=q_t.device)
    _need(out, torch.float32, "out", shape=(B, H, nT, nT))
    _check("veda_block_heat", lib().veda_block_heat(
        _ptr(q_t), _ptr(k_t), _ptr(maps.tile_valid), _ptr(lists.full_cnt), _ptr(lists.full_idx),
        _ptr(lists.part_cnt), _ptr(lists.part_idx), lists.stride, _ptr(lse), float(scale),
        _ptr(out), B, H, nT, D, _stream(stream)))
    return out


@dataclasses.dataclass
class MaskQuality:
    mass_rows: torch.Tensor     # [B, H, nT] heat kept per query tile
    recall_rows: torch.Tensor   # [B, H, nT] |pred & oracle| / |oracle|
    totals: torch.Tensor        # [4] see veda_mask_quality

    @property
    def mass(self) -> float:
        """Attention mass the mask keeps, over valid query slots."""
        t = self.totals.tolist()
        return t[0] / t[1] if t[1] else 0.0

    @property
    def recall(self) -> float:
        """Mean block recall against the oracle mask."""
        t = self.totals.tolist()
        return t[2] / t[3] if t[3] else 0.0


def mask_quality(heat: torch.Tensor, maps: DeviceMaps, pred: BlockLists, oracle: BlockLists,
                 stream=None) -> MaskQuality:
    """veda_mask_quality: kept attention mass of `pred` and its recall against `oracle`."""
    _need(heat, torch.float32, "heat")
    B, H, nT, nT2 = heat.shape
    if nT2 != nT:
        raise ValueError("heat: expected shape [B, H, nT, nT]")
    _need_maps(maps, H, nT * 128)
    _need_lists(pred, B, H, nT, "pred")
    _need_lists(oracle, B, H, nT, "oracle")
    dev = heat.device
    q = MaskQuality(torch.empty((B, H, nT), dtype=torch.float32, device=dev),
                    torch.empty((B, H, nT), dtype=torch.float32, device=dev),
                    torch.empty(4, dtype=torch.float32, device=dev))
    _check("veda_mask_quality", lib().veda_mask_quality(
        _ptr(heat), _ptr(maps.tile_valid), _ptr(maps.nT_per_head), _ptr(pred.full_cnt),
        _ptr(pred.full_idx), _ptr(pred.part_cnt), _ptr(pred.part_idx), pred.stride,
        _ptr(oracle.full_cnt), _ptr(oracle.full_idx), _ptr(oracle.part_cnt), _ptr(oracle.part_idx),
        oracle.stride, _ptr(q.mass_rows), _ptr(q.recall_rows), _ptr(q.totals), B, H, nT,
        _stream(stream)))
    return q


def rel_error(o: torch.Tensor, o_ref: torch.Tensor, stream=None) -> torch.Tensor:
    """veda_rel_error: [H, 2] sums of |o - o_ref|^2 and |o_ref|^2 per head (raster bf16)."""
    _need(o, torch.bfloat16, "o")
    _need(o_ref, torch.bfloat16, "o_ref", shape=o.shape)
    B, N, H, D = o.shape
    sums = torch.empty((H, 2), dtype=torch.float32, device=o.device)
    _check("veda_rel_error", lib().veda_rel_error(_ptr(o), _ptr(o_ref), _ptr(sums), B, N, H, D,
                                                  _stream(stream)))
    return sums


def tile_plan_vote(errors: np.ndarray, max_shapes: int = 2) -> Tuple[List[int], np.ndarray]:
    """veda_tile_plan_vote (host): the kept candidates (ascending) and each head's candidate
    from an [H, C] matrix of relative output errors."""
    err = np.ascontiguousarray(errors, dtype=np.float64)
    if err.ndim != 2:
        raise ValueError("errors: expected [H, C]")
    H, C = err.shape
    kept = np.zeros(max(1, min(max_shapes, C)), np.int32)
    n_kept = np.zeros(1, np.int32)
    assign = np.zeros(H, np.int32)
    _check("veda_tile_plan_vote", lib().veda_tile_plan_vote(
        err.ctypes.data, H, C, max_shapes, kept.ctypes.data, n_kept.ctypes.data, assign.ctypes.data))
    return [int(c) for c in kept[:int(n_kept[0])]], assign


def unpermute(o_t: torch.Tensor, maps: DeviceMaps, N: int, out: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    _need(o_t, torch.bfloat16, "o_tiled")
    B, H, Npad, D = o_t.shape
    _need_maps(maps, H, Npad)
    if out is None:
        out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=o_t.device)
    _need(out, torch.bfloat16, "out", shape=(B, N, H, D))
    _check("veda_unpermute", lib().veda_unpermute(
        _ptr(o_t), _ptr(out), _ptr(maps.tile_map), B, N, H, D, Npad, _stream(stream)))
    return out


def check_device_status(stream=None) -> int:
    """Synchronise the stream and raise if a kernel recorded an error. Returns the raw bits."""
    detail = ctypes.c_uint32(0)
    st = lib().veda_check_device_status(_stream(stream), ctypes.byref(detail))
    _check("veda_check_device_status", st)
    return detail.value


def selftest_wait_timeout(limit_us: int = 2000, stream=None) -> None:
    """Launch the bounded-wait self-test (see include/veda.h); check the status afterwards."""
    _check("veda_selftest_wait_timeout", lib().veda_selftest_wait_timeout(int(limit_us), _stream(stream)))


# ---------------------------------------------------------------------------------------
# the whole path
# ---------------------------------------------------------------------------------------

@dataclasses.dataclass
class PathBuffers:
    """Device buffers of one attention call (reusable across calls of the same shape)."""
    q_t: torch.Tensor
    k_t: torch.Tensor
    v_t: torch.Tensor
    pooled_q: torch.Tensor
    pooled_k: torch.Tensor
    scores: torch.Tensor
    workspace: torch.Tensor
    lists: BlockLists
    o_t: torch.Tensor
    lse: torch.Tensor
    o: torch.Tensor

    @staticmethod
    def allocate(B: int, N: int, H: int, maps: DeviceMaps, rho, device) -> "PathBuffers":
        nT, Npad, D = maps.nT, maps.Npad, 128
        bf = dict(dtype=torch.bfloat16, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        stride = list_stride_for(nT, rho)
        i32 = dict(dtype=torch.int32, device=device)
        lists = BlockLists(torch.zeros((B, H, nT), **i32), torch.zeros((B, H, nT, stride), **i32),
                           torch.zeros((B, H, nT), **i32), torch.zeros((B, H, nT, stride), **i32),
                           stride)
        return PathBuffers(
            torch.empty((B, H, Npad, D), **bf), torch.empty((B, H, Npad, D), **bf),
            torch.empty((B, H, Npad, D), **bf), torch.empty((B, H, nT, 3, D), **f32),
            torch.empty((B, H, nT, 3, D), **f32), torch.empty((B, H, nT, nT), **f32),
            torch.empty(block_scores_workspace_bytes(B, H, nT, D), dtype=torch.uint8, device=device),
            lists, torch.empty((B, H, Npad, D), **bf), torch.empty((B, H, Npad), **f32),
            torch.empty((B, N, H, D), **bf))


def sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, wq: torch.Tensor,
                     wk: torch.Tensor, maps: DeviceMaps, rho: Sequence[Tuple[int, int]],
                     scale: float, buffers: Optional[PathBuffers] = None, stream=None):
    """All six steps on raster Q/K/V [B, N, H, 128] (bf16, on the device).

    Returns the PathBuffers holding every intermediate; ``.o`` is the raster output. Steps 1
    and 2 of Q and K run as one call each (``permute_pool``: the tiles of ``permute_tiles``,
    the pooled features of ``tile_pool`` up to fp32 summation order in the mean), so that the
    tiled Q and K are not read a second time.
    """
    B, N, H, D = q.shape
    bufs = buffers or PathBuffers.allocate(B, N, H, maps, rho, q.device)
    permute_pool(q, maps, bufs.q_t, bufs.pooled_q, stream)
    permute_pool(k, maps, bufs.k_t, bufs.pooled_k, stream)
    permute_tiles(v, maps, bufs.v_t, stream)
    block_scores(bufs.pooled_q, bufs.pooled_k, wq, wk, bufs.scores, bufs.workspace, stream)
    select_blocks(bufs.scores, maps, rho, bufs.lists.stride, bufs.lists, stream)
    block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, bufs.lists, scale, bufs.o_t,
                          bufs.lse, stream=stream)
    unpermute(bufs.o_t, maps, N, bufs.o, stream)
    return bufs


class HostPipeline:
    """Clips from pinned host memory through the whole path, one clip per ``submit``.

    Three CUDA streams overlap the host-to-device copy of clip i + 1, the six steps of clip i
    and the device-to-host copy of clip i - 1's output (the host link carries both directions
    at once). Device copies of the raster inputs and of the raster output are kept per slot
    (``depth`` slots); CUDA events order every reuse of a slot after the work that last read
    it, so a clip's result does not depend on its neighbours. ``synchronize`` waits for every
    submitted clip's output to be in its host tensor.
    """

    def __init__(self, B: int, N: int, H: int, maps: DeviceMaps, rho: Sequence[Tuple[int, int]],
                 scale: float, device, depth: int = 2):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        self.maps, self.rho, self.scale, self.depth = maps, list(rho), float(scale), depth
        bf = dict(dtype=torch.bfloat16, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.inputs = [dict(q=torch.empty((B, N, H, 128), **bf), k=torch.empty((B, N, H, 128), **bf),
                            v=torch.empty((B, N, H, 128), **bf), wq=torch.empty((H, 128, 384), **f32),
                            wk=torch.empty((H, 128, 384), **f32)) for _ in range(depth)]
        self.outputs = [torch.empty((B, N, H, 128), **bf) for _ in range(depth)]
        self.bufs = PathBuffers.allocate(B, N, H, maps, rho, device)
        self.h2d, self.comp, self.d2h = (torch.cuda.Stream(device) for _ in range(3))
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]
        self.in_ready, self.in_free, self.out_ready, self.out_free = ev(), ev(), ev(), ev()
        self.n = 0

    def submit(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, wq: torch.Tensor, wk: torch.Tensor,
               out: torch.Tensor) -> None:
        """Enqueue one clip: q / k / v [B, N, H, 128] bf16, wq / wk [H, 128, 384] fp32 and the
        output out [B, N, H, 128] bf16, all pinned host tensors; returns at once."""
        s = self.n % self.depth
        reuse = self.n >= self.depth
        slot = self.inputs[s]
        # inputs of slot s: after the clip that last used them has been computed
        if reuse:
            self.h2d.wait_event(self.in_free[s])
        with torch.cuda.stream(self.h2d):
            for name, src in (("q", q), ("k", k), ("v", v), ("wq", wq), ("wk", wk)):
                slot[name].copy_(src, non_blocking=True)
            self.in_ready[s].record(self.h2d)
        # the six steps, into output slot s once its previous contents have left the device
        self.comp.wait_event(self.in_ready[s])
        if reuse:
            self.comp.wait_event(self.out_free[s])
        bufs = dataclasses.replace(self.bufs, o=self.outputs[s])
        sparse_attention(slot["q"], slot["k"], slot["v"], slot["wq"], slot["wk"], self.maps, self.rho,
                         self.scale, buffers=bufs, stream=self.comp)
        self.in_free[s].record(self.comp)
        self.out_ready[s].record(self.comp)
        # the output of slot s to the host
        self.d2h.wait_event(self.out_ready[s])
        with torch.cuda.stream(self.d2h):
            out.copy_(self.outputs[s], non_blocking=True)
            self.out_free[s].record(self.d2h)
        self.n += 1

    def synchronize(self) -> None:
        self.d2h.synchronize()
