"""Thin Python binding of libaq's C ABI (include/aq.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libaq.so.  PyTorch provides device memory and the current CUDA
stream.  There is no CPU fallback: if libaq.so is missing the first call
raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libaq.so")

AQ_OK = 0
AQ_F32, AQ_BF16 = 0, 1
AQ_PHASE_DECODE, AQ_PHASE_PREFILL = 0, 1
BUF_NAMES = ("bitmap", "row_off4", "row_off8", "tile_idx", "w4", "w8", "scales")
EXPORTED = ("aq_status_str", "aq_packed_sizes", "aq_pack_metadata", "aq_pack", "aq_quant_act",
            "aq_workspace_bytes", "aq_linear_decode", "aq_linear_prefill", "aq_debug_tile_partials",
            "aq_linear_group", "aq_group_workspace_bytes", "aq_workspace_status", "aq_linear_decode_noalloc",
            "aq_quantize_weights", "aq_paper_packed_bytes", "aq_expanded_bytes", "aq_expand_int8",
            "aq_linear_prefill_expanded", "aq_act_group_rows", "aq_quant_act_groups", "aq_measure_i8_peak",
            "aq_debug_linear_stalled", "aq_pack_tiles", "aq_paper_quant_act", "aq_paper_linear",
            "aq_debug_paper_partials")


class AqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().aq_status_str(status).decode()} ({status})")


AQ_SCALES_ROW_FP16, AQ_SCALES_TILE_FP32 = 0, 1


class AqPackedStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("N", "K", "bN", "bK", "R", "C", "T4", "T8")] + \
               [(n, ctypes.c_void_p) for n in BUF_NAMES] + [("scale_kind", ctypes.c_int32)]


_lib = None


def lib():
    """Load libaq.so once and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m w8_a8_quantized_b200.build` "
                           "(this package has no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    c_int, c_void_p, c_size_t = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    P = ctypes.POINTER(AqPackedStruct)
    L.aq_status_str.restype = ctypes.c_char_p
    L.aq_status_str.argtypes = [c_int]
    L.aq_packed_sizes.restype = c_int
    L.aq_packed_sizes.argtypes = [c_int, c_int, c_int, c_int, c_int, ctypes.POINTER(c_size_t)]
    L.aq_pack_metadata.restype = c_int
    L.aq_pack_metadata.argtypes = [c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                   ctypes.POINTER(ctypes.c_int32)]
    L.aq_pack.restype = c_int
    L.aq_pack.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, P, c_void_p]
    L.aq_pack_tiles.restype = c_int
    L.aq_pack_tiles.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, P, c_void_p]
    L.aq_paper_quant_act.restype = c_int
    L.aq_paper_quant_act.argtypes = [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]
    L.aq_paper_linear.restype = c_int
    L.aq_paper_linear.argtypes = [P, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_int, c_void_p]
    L.aq_debug_paper_partials.restype = c_int
    L.aq_debug_paper_partials.argtypes = [P, c_void_p, c_int, c_void_p, c_void_p]
    L.aq_quant_act.restype = c_int
    L.aq_paper_packed_bytes.restype = c_int
    L.aq_paper_packed_bytes.argtypes = [c_int, c_int, c_int, c_int, c_int, ctypes.POINTER(c_size_t)]
    L.aq_expanded_bytes.restype = c_size_t
    L.aq_expanded_bytes.argtypes = [P]
    L.aq_expand_int8.restype = c_int
    L.aq_expand_int8.argtypes = [P, c_void_p, c_size_t, P, c_void_p]
    L.aq_linear_prefill_expanded.restype = c_int
    L.aq_linear_prefill_expanded.argtypes = [P, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p,
                                             c_size_t, c_void_p, c_size_t, c_void_p]
    L.aq_act_group_rows.restype = c_int
    L.aq_act_group_rows.argtypes = [c_int]
    L.aq_quant_act_groups.restype = c_int
    L.aq_quant_act_groups.argtypes = [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]
    L.aq_quantize_weights.restype = c_int
    L.aq_quantize_weights.argtypes = [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_int,
                                      c_void_p, c_void_p, c_void_p]
    L.aq_quant_act.argtypes = [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]
    L.aq_workspace_bytes.restype = c_size_t
    L.aq_workspace_bytes.argtypes = [c_int, c_int, P]
    for f in (L.aq_linear_decode, L.aq_linear_prefill):
        f.restype = c_int
        f.argtypes = [P, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p, c_size_t,
                      c_void_p]
    L.aq_debug_tile_partials.restype = c_int
    L.aq_debug_tile_partials.argtypes = [P, c_void_p, c_int, c_int, c_void_p, c_void_p, c_size_t, c_void_p]
    L.aq_linear_group.restype = c_int
    L.aq_linear_group.argtypes = [c_int, ctypes.POINTER(P), c_int, c_void_p, c_int, c_int, ctypes.POINTER(c_void_p),
                                  ctypes.POINTER(c_void_p), ctypes.POINTER(c_int), c_int, c_void_p, c_size_t,
                                  c_void_p]
    L.aq_group_workspace_bytes.restype = c_size_t
    L.aq_group_workspace_bytes.argtypes = [c_int, c_int, ctypes.POINTER(P), c_int]
    L.aq_linear_decode_noalloc.restype = c_int
    L.aq_linear_decode_noalloc.argtypes = [P, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p]
    L.aq_debug_linear_stalled.restype = c_int
    L.aq_debug_linear_stalled.argtypes = [P, c_void_p, c_void_p, c_int, c_int, c_void_p, c_int, c_void_p, c_size_t,
                                          ctypes.c_ulonglong, c_int, c_void_p]
    L.aq_measure_i8_peak.restype = c_int
    L.aq_measure_i8_peak.argtypes = [c_int, ctypes.POINTER(ctypes.c_double), c_void_p]
    L.aq_workspace_status.restype = c_int
    L.aq_workspace_status.argtypes = [c_void_p, c_void_p, ctypes.POINTER(c_int)]
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != AQ_OK:
        raise AqError(rc, what)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype, device=None):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError(f"{name} must be a {dtype} tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def aq_packed_sizes(N: int, K: int, bN: int, bK: int, T4: int) -> dict:
    out = (ctypes.c_size_t * 7)()
    _check(lib().aq_packed_sizes(N, K, bN, bK, T4, out), "aq_packed_sizes")
    return dict(zip(BUF_NAMES, [int(v) for v in out]))


def aq_paper_packed_bytes(R: int, C: int, T4: int, bN: int, bK: int) -> int:
    """Storage of one packed projection as eq. 18 accounts it (FP32 scale per tile)."""
    out = ctypes.c_size_t()
    _check(lib().aq_paper_packed_bytes(R, C, T4, bN, bK, ctypes.byref(out)), "aq_paper_packed_bytes")
    return int(out.value)


class PackedWeights:
    """Device buffers of one packed projection plus the C struct describing them."""

    def __init__(self, N: int, K: int, bN: int, bK: int, T4: int, device):
        sizes = aq_packed_sizes(N, K, bN, bK, T4)
        self.device = torch.device(device)
        self.buffers = {n: torch.empty(max(s, 16), dtype=torch.uint8, device=self.device) for n, s in sizes.items()}
        self.sizes = sizes
        self.struct = AqPackedStruct(N=N, K=K, bN=bN, bK=bK, R=N // bN, C=K // bK, T4=T4, T8=0)
        for n in BUF_NAMES:
            setattr(self.struct, n, self.buffers[n].data_ptr())

    N = property(lambda s: s.struct.N)
    K = property(lambda s: s.struct.K)
    bN = property(lambda s: s.struct.bN)
    bK = property(lambda s: s.struct.bK)
    R = property(lambda s: s.struct.R)
    C = property(lambda s: s.struct.C)
    T4 = property(lambda s: s.struct.T4)
    T8 = property(lambda s: s.struct.T8)

    @property
    def nbytes(self) -> int:
        """Bytes of the packed representation (all seven buffers)."""
        return sum(self.sizes.values())

    def host_buffers(self) -> dict:
        return {n: self.buffers[n][: self.sizes[n]].cpu().numpy() for n in BUF_NAMES}


def aq_pack(codes: torch.Tensor, scales: torch.Tensor, pmap: torch.Tensor, bN: int, bK: int) -> PackedWeights:
    """codes int8 [N][K], scales float16 [N][C], pmap uint8 [R][C] (1 = INT4), all on one CUDA device."""
    _need(codes, "codes", torch.int8)
    dev = codes.device
    _need(scales, "scales", torch.float16, dev)
    _need(pmap, "pmap", torch.uint8, dev)
    N, K = codes.shape
    T4 = aq_int4_tiles(pmap)
    if scales.dim() != 2 or scales.shape[0] != N or pmap.dim() != 2 or pmap.shape[0] * bN != N or \
            pmap.shape[1] * bK != K or scales.shape[1] != pmap.shape[1]:
        raise ValueError("codes [N][K], scales [N][C] and pmap [R][C] do not agree with the tile shape")
    w = PackedWeights(N, K, bN, bK, T4, dev)
    with torch.cuda.device(dev):
        _check(lib().aq_pack(codes.data_ptr(), scales.data_ptr(), pmap.data_ptr(), N, K, bN, bK,
                             ctypes.byref(w.struct), _stream(dev)), "aq_pack")
    return w


def aq_pack_tiles(codes: torch.Tensor, tile_scales: torch.Tensor, pmap: torch.Tensor, bN: int,
                  bK: int = 64) -> PackedWeights:
    """Paper-exact packing: codes int8 [N][K], tile_scales float32 [R][C] (one
    scale per whole tile), pmap uint8 [R][C] (1 = INT4), bK = 64."""
    _need(codes, "codes", torch.int8)
    dev = codes.device
    _need(tile_scales, "tile_scales", torch.float32, dev)
    _need(pmap, "pmap", torch.uint8, dev)
    N, K = codes.shape
    if pmap.dim() != 2 or pmap.shape[0] * bN != N or pmap.shape[1] * bK != K or \
            tuple(tile_scales.shape) != tuple(pmap.shape):
        raise ValueError("codes [N][K], tile_scales [R][C] and pmap [R][C] do not agree with the tile shape")
    T4 = aq_int4_tiles(pmap)
    w = PackedWeights(N, K, bN, bK, T4, dev)
    with torch.cuda.device(dev):
        _check(lib().aq_pack_tiles(codes.data_ptr(), tile_scales.data_ptr(), pmap.data_ptr(), N, K, bN, bK,
                                   ctypes.byref(w.struct), _stream(dev)), "aq_pack_tiles")
    return w


def aq_paper_quant_act(x: torch.Tensor, v: torch.Tensor = None):
    """Paper-exact activation preparation: x bf16 [M][ldx], v float32 [K/64][64][64]
    (V_c blocks; None = identity) -> (xq int8 [M'][K], sx float32 [M'/b_M][K/64])."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 CUDA tensor with unit inner stride")
    M, K = x.shape
    if v is not None:
        _need(v, "v", torch.float32, x.device)
        if tuple(v.shape) != (K // 64, 64, 64):
            raise ValueError("v must be float32 [K/64][64][64]")
    bM = int(lib().aq_act_group_rows(M))
    Mp = -(-M // bM) * bM
    xq = torch.empty((Mp, K), dtype=torch.int8, device=x.device)
    sx = torch.empty((Mp // bM, max(K // 64, 1)), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        _check(lib().aq_paper_quant_act(x.data_ptr(), M, K, x.stride(0), v.data_ptr() if v is not None else None,
                                        xq.data_ptr(), sx.data_ptr(), _stream(x.device)), "aq_paper_quant_act")
    return xq, sx


def _paper_operands(w: PackedWeights, xq: torch.Tensor, M: int) -> int:
    """Check the paper-exact layer's codes against the packed weights: the kernel
    reads xq as [M'][K] (M' = M rounded up to whole row groups); returns the
    number of activation row groups M' / b_M."""
    if w.struct.scale_kind != AQ_SCALES_TILE_FP32:
        raise ValueError("w must be packed by aq_pack_tiles (per-tile fp32 scales)")
    _need(xq, "xq", torch.int8, w.device)
    bM = int(lib().aq_act_group_rows(M)) if M >= 1 else 0
    if bM == 0:
        raise ValueError("M must be at least 1")
    Mp = -(-M // bM) * bM
    if xq.dim() != 2 or xq.shape[1] != w.K or xq.shape[0] < Mp:
        raise ValueError(f"xq must be [>= {Mp}][{w.K}] (M = {M} padded to whole row groups), got {tuple(xq.shape)}")
    return Mp // bM


def aq_paper_linear(w: PackedWeights, xq: torch.Tensor, sx: torch.Tensor, M: int, u: torch.Tensor = None,
                    bias: torch.Tensor = None, out: torch.Tensor = None) -> torch.Tensor:
    """Paper-exact layer (eq. 19, then Y = Y~ U): w from aq_pack_tiles, (xq, sx)
    from aq_paper_quant_act, u float32 [R][bN][bN] (None = identity), bias
    float32 [N] -> y float32 [M][N]."""
    dev = w.device
    groups = _paper_operands(w, xq, M)
    _need(sx, "sx", torch.float32, dev)
    if sx.numel() < groups * w.C:
        raise ValueError(f"sx must hold [{groups}][{w.C}] group scales, got {sx.numel()} values")
    if u is not None:
        _need(u, "u", torch.float32, dev)
        if tuple(u.shape) != (w.R, w.bN, w.bN):
            raise ValueError("u must be float32 [R][bN][bN]")
    if bias is not None:
        _need(bias, "bias", torch.float32, dev)
        if bias.numel() != w.N:
            raise ValueError("bias must have N elements")
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    if out.dim() != 2 or out.shape[0] < M or out.shape[1] < w.N or out.stride(1) != 1:
        raise ValueError("out must be float32 [>= M][>= N] with unit inner stride")
    with torch.cuda.device(dev):
        _check(lib().aq_paper_linear(ctypes.byref(w.struct), xq.data_ptr(), sx.data_ptr(), M,
                                     u.data_ptr() if u is not None else None,
                                     bias.data_ptr() if bias is not None else None, out.data_ptr(), out.stride(0),
                                     _stream(dev)), "aq_paper_linear")
    return out


def aq_debug_paper_partials(w: PackedWeights, xq: torch.Tensor, M: int) -> torch.Tensor:
    """Exact integer tile products of the paper-exact layer: int32 [M][N][K/64]."""
    dev = w.device
    _paper_operands(w, xq, M)
    P = torch.zeros((M, w.N, w.C), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().aq_debug_paper_partials(ctypes.byref(w.struct), xq.data_ptr(), M, P.data_ptr(), _stream(dev)),
               "aq_debug_paper_partials")
    return P


def aq_int4_tiles(pmap: torch.Tensor) -> int:
    """INT4 tile count of a precision map (uint8 [R][C], 1 = INT4), as the library's
    host-side metadata builder counts it; it rejects labels other than 0 and 1."""
    if pmap.dim() != 2 or pmap.dtype != torch.uint8:
        raise ValueError("pmap must be a 2-D uint8 tensor")
    R, C = pmap.shape
    host = np.ascontiguousarray(pmap.cpu().numpy())
    T = R * C
    bitmap = np.zeros(max((T + 7) // 8, 1), np.uint8)
    off4, off8 = np.zeros(R + 1, np.int32), np.zeros(R + 1, np.int32)
    idx = np.zeros(max(T, 1), np.int32)
    t4 = ctypes.c_int32(0)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().aq_pack_metadata(p(host), R, C, p(bitmap), p(off4), p(off8), p(idx), ctypes.byref(t4)),
           "aq_pack_metadata")
    return int(t4.value)


def aq_quantize_weights(w: torch.Tensor, pmap: torch.Tensor, bN: int, bK: int = 128, search: bool = True,
                        codes: torch.Tensor = None, scales: torch.Tensor = None):
    """Float weights w (float32 or bfloat16, [N][ldw] with unit inner stride) and
    labels pmap uint8 [R][C] (1 = INT4) -> (codes int8 [N][K], scales float16
    [N][C]) for aq_pack.  K = pmap.shape[1] * bK; search selects eq. 7's scale
    search over eq. 6's endpoint scale."""
    if w.dim() != 2 or not w.is_cuda or w.stride(1) != 1 or w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("w must be a 2-D float32 or bfloat16 CUDA tensor with unit inner stride")
    dev = w.device
    _need(pmap, "pmap", torch.uint8, dev)
    N, K = w.shape[0], pmap.shape[1] * bK
    if codes is None:
        codes = torch.empty((N, K), dtype=torch.int8, device=dev)
    if scales is None:
        scales = torch.empty((N, pmap.shape[1]), dtype=torch.float16, device=dev)
    _need(codes, "codes", torch.int8, dev)
    _need(scales, "scales", torch.float16, dev)
    wdtype = AQ_F32 if w.dtype == torch.float32 else AQ_BF16
    _check(lib().aq_quantize_weights(w.data_ptr(), wdtype, N, K, w.stride(0), bN, bK, pmap.data_ptr(),
                                     int(bool(search)), codes.data_ptr(), scales.data_ptr(), _stream(dev)),
           "aq_quantize_weights")
    return codes, scales


def aq_quantize_and_pack(w: torch.Tensor, pmap: torch.Tensor, bN: int, bK: int = 128,
                         search: bool = True) -> PackedWeights:
    """Float weights -> packed tile format: aq_quantize_weights then aq_pack."""
    codes, scales = aq_quantize_weights(w, pmap, bN, bK, search)
    return aq_pack(codes, scales, pmap, bN, bK)


def aq_quant_act(x: torch.Tensor, xq: torch.Tensor = None, sx: torch.Tensor = None, K: int = None):
    """x bf16 [M][ldx] -> (xq int8 [M][K], sx float32 [M]) on x's stream."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 CUDA tensor with unit inner stride")
    M = x.shape[0]
    K = x.shape[1] if K is None else K
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need(xq, "xq", torch.int8, x.device)
    _need(sx, "sx", torch.float32, x.device)
    if xq.dim() != 2 or xq.shape[0] < M or xq.shape[1] != K or sx.numel() < M or x.shape[1] < K:
        raise ValueError("xq must be [M][K] and sx hold M scales, with K <= x.shape[1]")
    with torch.cuda.device(x.device):
        _check(lib().aq_quant_act(x.data_ptr(), M, K, x.stride(0), xq.data_ptr(), sx.data_ptr(),
                                  _stream(x.device)), "aq_quant_act")
    return xq, sx


def aq_quant_act_groups(x: torch.Tensor, K: int = None):
    """Paper-form activation quantization: x bf16 [M][ldx] -> (xq int8 [M'][K],
    sx float32 [M'/b_M][K/64]) with one scale per 64 features x b_M rows."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 CUDA tensor with unit inner stride")
    M = x.shape[0]
    K = x.shape[1] if K is None else K
    bM = int(lib().aq_act_group_rows(M))
    Mp = -(-M // bM) * bM
    xq = torch.empty((Mp, K), dtype=torch.int8, device=x.device)
    sx = torch.empty((Mp // bM, K // 64), dtype=torch.float32, device=x.device)
    _check(lib().aq_quant_act_groups(x.data_ptr(), M, K, x.stride(0), xq.data_ptr(), sx.data_ptr(),
                                     _stream(x.device)), "aq_quant_act_groups")
    return xq, sx


def aq_workspace_bytes(phase: int, M: int, w: PackedWeights) -> int:
    return int(lib().aq_workspace_bytes(phase, M, ctypes.byref(w.struct)))


_ws_cache = {}


def workspace(phase: int, M: int, w: PackedWeights) -> torch.Tensor:
    """A zero-initialised workspace big enough for (phase, M, w), cached per device."""
    need = aq_workspace_bytes(phase, M, w)
    if need == 0:
        raise ValueError("invalid arguments for a workspace")
    key = (w.device, phase)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=w.device)
        _ws_cache[key] = ws
    return ws


def _linear_operands(w, xq, sx, bias, out, out_dtype):
    """Check the operands of a linear call against the packed weights (shapes the
    kernels read and write through raw pointers); allocate `out` if absent."""
    _need(xq, "xq", torch.int8, w.device)
    _need(sx, "sx", torch.float32, w.device)
    if xq.dim() != 2 or xq.shape[1] != w.K:
        raise ValueError(f"xq must be [M][{w.K}], got {tuple(xq.shape)}")
    M = xq.shape[0]
    if M < 1 or sx.numel() < M:
        raise ValueError(f"sx must hold at least M = {M} token scales")
    if out is None:
        out = torch.empty((M, w.N), dtype=out_dtype, device=w.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or out.dim() != 2 or out.stride(1) != 1 or \
            out.device != w.device:
        raise ValueError("out must be a 2-D float32 or bfloat16 tensor on the weights' device, unit inner stride")
    if out.shape[0] < M or out.shape[1] < w.N:
        raise ValueError(f"out must be at least [{M}][{w.N}], got {tuple(out.shape)}")
    if bias is not None:
        _need(bias, "bias", torch.float32, w.device)
        if bias.numel() < w.N:
            raise ValueError(f"bias must hold N = {w.N} values")
    return M, out


def _linear(fn, name, phase, w, xq, sx, bias, out, out_dtype, ws):
    M, out = _linear_operands(w, xq, sx, bias, out, out_dtype)
    ydt = AQ_F32 if out.dtype == torch.float32 else AQ_BF16
    if ws is None:
        ws = workspace(phase, M, w)
    with torch.cuda.device(w.device):
        _check(fn(ctypes.byref(w.struct), xq.data_ptr(), sx.data_ptr(), M,
                  bias.data_ptr() if bias is not None else None, out.data_ptr(), ydt, out.stride(0),
                  ws.data_ptr(), ws.numel(), _stream(w.device)), name)
    return out


def aq_linear_decode(w: PackedWeights, xq, sx, bias=None, out=None, out_dtype=torch.float32, ws=None):
    """Decode-phase y = sx * sum_j sw * (xq q^T)_j (+ bias) for 1 <= M <= 64 tokens."""
    return _linear(lib().aq_linear_decode, "aq_linear_decode", AQ_PHASE_DECODE, w, xq, sx, bias, out, out_dtype, ws)


def aq_linear_prefill(w: PackedWeights, xq, sx, bias=None, out=None, out_dtype=torch.float32, ws=None):
    """Prefill-phase y (tensor-core INT8 path), any M >= 1."""
    return _linear(lib().aq_linear_prefill, "aq_linear_prefill", AQ_PHASE_PREFILL, w, xq, sx, bias, out, out_dtype,
                   ws)


def aq_expanded_bytes(w: PackedWeights) -> int:
    """Bytes of the all-INT8 copy of w made by the long-prefill variant."""
    return int(lib().aq_expanded_bytes(ctypes.byref(w.struct)))


class ExpandedWeights:
    """The all-INT8 copy of a packed projection (long-prefill variant); shares w's scales."""

    def __init__(self, w: PackedWeights, buf: torch.Tensor = None):
        need = aq_expanded_bytes(w)
        if need == 0:
            raise ValueError("invalid packed weights")
        self.source, self.device = w, w.device
        self.buf = torch.empty(need + 256, dtype=torch.uint8, device=w.device) if buf is None else buf
        off = (-self.buf.data_ptr()) % 256  # the library wants a 256-byte aligned buffer
        self.base = self.buf[off:off + need]
        self.struct = AqPackedStruct()
        _check(lib().aq_expand_int8(ctypes.byref(w.struct), self.base.data_ptr(), need, ctypes.byref(self.struct),
                                    _stream(w.device)), "aq_expand_int8")

    N = property(lambda s: s.struct.N)
    K = property(lambda s: s.struct.K)
    R = property(lambda s: s.struct.R)
    C = property(lambda s: s.struct.C)
    T4 = property(lambda s: s.struct.T4)
    T8 = property(lambda s: s.struct.T8)

    def host_buffers(self) -> dict:
        """Bitmap, offsets, tile table and INT8 payload as host arrays (scales: the source's)."""
        st, R, C, bN = self.struct, self.R, self.C, self.struct.bN
        T = R * C
        def view(ptr, nbytes):
            o = ptr - self.base.data_ptr()
            return self.base[o:o + nbytes].cpu().numpy()
        return {"bitmap": view(st.bitmap, (T + 7) // 8), "row_off4": view(st.row_off4, 4 * (R + 1)).view(np.int32),
                "row_off8": view(st.row_off8, 4 * (R + 1)).view(np.int32),
                "tile_idx": view(st.tile_idx, 4 * T).view(np.int32),
                "w8": view(st.w8, T * bN * 128).view(np.int8).reshape(T, bN, 128)}


def aq_linear_prefill_expanded(w: PackedWeights, xq, sx, bias=None, out=None, out_dtype=torch.float32, ws=None,
                               tmp=None):
    """aq_linear_prefill through the long-prefill variant: expand to an INT8 copy in
    `tmp` (uint8, >= aq_expanded_bytes(w) + 256), then the pure INT8 GEMM."""
    need = aq_expanded_bytes(w)
    if tmp is None:
        tmp = torch.empty(need + 256, dtype=torch.uint8, device=w.device)
    off = (-tmp.data_ptr()) % 256
    if tmp.numel() - off < need:
        raise ValueError("tmp is too small")
    L = lib()
    def fn(wp, xqp, sxp, M, bp, yp, ydt, ldy, wsp, wsn, st):
        return L.aq_linear_prefill_expanded(wp, xqp, sxp, M, bp, yp, ydt, ldy, wsp, wsn, tmp.data_ptr() + off,
                                            tmp.numel() - off, st)
    return _linear(fn, "aq_linear_prefill_expanded", AQ_PHASE_PREFILL, w, xq, sx, bias, out, out_dtype, ws)


def aq_linear_decode_noalloc(w: PackedWeights, xq, sx, bias=None, out=None, out_dtype=torch.float32):
    """aq_linear_decode without a workspace, for callers that cannot allocate device
    memory: the library's fixed 4 MiB device scratch is used instead (calls that
    overlap on the GPU must not share it).  `out` must be preallocated by callers
    that cannot allocate; it is allocated here only for convenience."""
    M, out = _linear_operands(w, xq, sx, bias, out, out_dtype)
    # the library resolves its scratch array on the CURRENT device: make it the weights' device
    with torch.cuda.device(w.device):
        _check(lib().aq_linear_decode_noalloc(ctypes.byref(w.struct), xq.data_ptr(), sx.data_ptr(), M,
                                              bias.data_ptr() if bias is not None else None, out.data_ptr(),
                                              AQ_F32 if out.dtype == torch.float32 else AQ_BF16, out.stride(0),
                                              _stream(w.device)), "aq_linear_decode_noalloc")
    return out


class Group:
    """Projections sharing one input (q/k/v or gate/up), run by aq_linear_group."""

    def __init__(self, weights, phase: int, M: int):
        self.weights = list(weights)
        self.phase, self.M = phase, M
        G = len(self.weights)
        P = ctypes.POINTER(AqPackedStruct)
        self._w = (P * G)(*[ctypes.pointer(w.struct) for w in self.weights])
        need = int(lib().aq_group_workspace_bytes(phase, M, self._w, G))
        if need == 0:
            raise ValueError("invalid projection group")
        self.ws = torch.zeros(need, dtype=torch.uint8, device=self.weights[0].device)

    def __call__(self, x: torch.Tensor, outs, bias=None, ws=None):
        """x bf16 [M][ldx]; outs: one float32 or bfloat16 [M][N_g] tensor per member."""
        G = len(self.weights)
        dev = self.weights[0].device
        if x.dtype != torch.bfloat16 or x.device != dev or x.dim() != 2 or x.stride(1) != 1:
            raise ValueError("x must be a 2-D bf16 tensor on the weights' device with unit inner stride")
        if x.shape[0] != self.M or x.shape[1] < self.weights[0].K or len(outs) != G:
            raise ValueError("token count, input width or number of outputs does not match the group")
        for o, w in zip(outs, self.weights):
            if o.dim() != 2 or o.shape[0] < self.M or o.shape[1] < w.N:
                raise ValueError(f"each output must be at least [M][N] = [{self.M}][{w.N}]")
        if bias is not None and (len(bias) != G or any(b is not None and (b.dtype != torch.float32 or
                                                                       b.device != dev or b.numel() < w.N or
                                                                       not b.is_contiguous())
                                                      for b, w in zip(bias, self.weights))):
            raise ValueError("bias must hold one contiguous float32 [N] tensor (or None) per member")
        dt = outs[0].dtype
        if dt not in (torch.float32, torch.bfloat16) or any(o.dtype != dt or o.device != dev or o.stride(1) != 1
                                                             for o in outs):
            raise ValueError("outputs must share one dtype (float32 or bfloat16) on the weights' device")
        ys = (ctypes.c_void_p * G)(*[o.data_ptr() for o in outs])
        lds = (ctypes.c_int * G)(*[o.stride(0) for o in outs])
        bs = None
        if bias is not None:
            bs = (ctypes.c_void_p * G)(*[b.data_ptr() if b is not None else None for b in bias])
        ws = self.ws if ws is None else ws
        ydt = AQ_F32 if dt == torch.float32 else AQ_BF16
        with torch.cuda.device(dev):
            _check(lib().aq_linear_group(self.phase, self._w, G, x.data_ptr(), x.stride(0), self.M, bs, ys, lds,
                                         ydt, ws.data_ptr(), ws.numel(), _stream(dev)), "aq_linear_group")
        return outs


def aq_debug_tile_partials(w: PackedWeights, xq: torch.Tensor, phase: int, ws=None) -> torch.Tensor:
    """Exact INT32 tile products P[M][N][C] computed by the `phase` data path."""
    _need(xq, "xq", torch.int8, w.device)
    if xq.dim() != 2 or xq.shape[1] != w.K:
        raise ValueError(f"xq must be [M][{w.K}]")
    M = xq.shape[0]
    P = torch.zeros((M, w.N, w.C), dtype=torch.int32, device=w.device)
    if ws is None:
        ws = workspace(AQ_PHASE_PREFILL, M, w)
    with torch.cuda.device(w.device):
        _check(lib().aq_debug_tile_partials(ctypes.byref(w.struct), xq.data_ptr(), M, phase, P.data_ptr(),
                                            ws.data_ptr(), ws.numel(), _stream(w.device)), "aq_debug_tile_partials")
    return P


def aq_debug_linear_stalled(w: PackedWeights, xq, sx, phase: int, ws: torch.Tensor, wait_ns: int = 20_000_000,
                            stop_after: int = 1) -> torch.Tensor:
    """Run the tensor-core linear kernel with a stage that never fills (test of the
    bounded waits): returns the (unspecified) output; the error lands in `ws`."""
    M, out = _linear_operands(w, xq, sx, None, None, torch.float32)
    with torch.cuda.device(w.device):
        _check(lib().aq_debug_linear_stalled(ctypes.byref(w.struct), xq.data_ptr(), sx.data_ptr(), M, phase,
                                             out.data_ptr(), out.stride(0), ws.data_ptr(), ws.numel(), wait_ns,
                                             stop_after, _stream(w.device)), "aq_debug_linear_stalled")
    return out


def aq_workspace_status(ws: torch.Tensor):
    """Synchronise; return (status, info) of the kernel error word of a workspace and clear it."""
    info = ctypes.c_int(0)
    rc = lib().aq_workspace_status(ws.data_ptr(), _stream(ws.device), ctypes.byref(info))
    if rc not in (AQ_OK, -7):
        _check(rc, "aq_workspace_status")
    return rc, info.value


def aq_measure_i8_peak(iters: int = 20000, device=None) -> float:
    """Measured dense INT8 tensor-core rate of the device in TOPS (tcgen05 loop on
    shared-memory operands; a measurement helper, not part of the layer)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    tops = ctypes.c_double(0.0)
    with torch.cuda.device(dev):
        _check(lib().aq_measure_i8_peak(iters, ctypes.byref(tops), _stream(dev)), "aq_measure_i8_peak")
    return float(tops.value)


def check_all_workspaces():
    """Raise if any cached workspace recorded a kernel error."""
    for ws in _ws_cache.values():
        rc, info = aq_workspace_status(ws)
        if rc != AQ_OK:
            raise AqError(rc, f"kernel wait gave up (info {info})")
