"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/aq.h declares, and its host-only logic (buffer sizing, packed-format
metadata, argument validation) agrees with the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from w8_a8_quantized_b200 import aq, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "aq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(aq_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("aq_pack", "aq_quant_act", "aq_linear_decode", "aq_linear_prefill"):
        assert required in names
    assert set(names) == set(aq.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = aq.lib()
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_binding_argument_counts_match_the_header():
    """Every declaration's parameter count equals the length of the binding's
    ctypes argtypes for it (a missing or extra argument would be marshalled
    silently)."""
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "aq.h")).read(), flags=re.S)
    decls = dict(re.findall(r"\b(aq_\w+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S))
    assert set(decls) == set(_declared_functions())
    L = aq.lib()
    c_scalars = {"int": (ctypes.c_int, False), "size_t": (ctypes.c_size_t, False),
                 "unsigned long long": (ctypes.c_ulonglong, False), "double": (ctypes.c_double, True)}
    for name, params in decls.items():
        ps = [] if params.strip() in ("", "void") else params.split(",")
        argtypes = getattr(L, name).argtypes
        assert argtypes is not None and len(argtypes) == len(ps), name
        for p, t in zip(ps, argtypes):  # pointer-ness, then width and int / float class of scalars
            is_ptr = t in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(t, ctypes._Pointer)
            assert ("*" in p) == is_ptr, (name, p)
            if not is_ptr:
                want, is_float = c_scalars[" ".join(p.split()[:-1]).replace("const ", "")]
                assert ctypes.sizeof(t) == ctypes.sizeof(want), (name, p)
                assert issubclass(t, (ctypes.c_double, ctypes.c_float)) == is_float, (name, p)


def test_packed_struct_layout_matches_the_header():
    """AqPackedStruct lists aq_packed's fields in the header's order, with the
    same widths (int32 scalars, pointers)."""
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "aq.h")).read(), flags=re.S)
    body = re.search(r"typedef struct aq_packed \{(.*?)\} aq_packed;", src, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        ctype, names = decl.split(None, 1)
        ptr = ctype.endswith("*") or names.startswith("*")
        for n in names.replace("*", "").split(","):
            fields.append((n.strip(), ptr, ctype.rstrip("*")))
    py = aq.AqPackedStruct._fields_
    assert [f[0] for f in fields] == [n for n, _ in py]
    for (name, ptr, ctype), (_, t) in zip(fields, py):
        assert (t is ctypes.c_void_p) == ptr, name
        if not ptr:
            assert ctype == "int32_t" and t is ctypes.c_int32, name


def test_status_strings():
    L = aq.lib()
    for code in range(0, -8, -1):
        assert L.aq_status_str(code).decode().startswith("AQ_")
    assert L.aq_status_str(12345).decode() == "unknown aq_status"


@pytest.mark.parametrize("N,K,bN,T4", [(256, 512, 128, 3), (192, 384, 64, 0), (128, 128, 128, 1), (5120, 17408, 128, 3000)])
def test_packed_sizes_match_oracle(N, K, bN, T4):
    sz = aq.aq_packed_sizes(N, K, bN, 128, T4)
    R, C = N // bN, K // 128
    g = dict(N=N, bN=bN, bK=128, R=R, C=C, T4=T4, T8=R * C - T4)
    assert sum(sz.values()) == oracle.packed_bytes(g)
    assert sz["w4"] == T4 * bN * 64 and sz["w8"] == (R * C - T4) * bN * 128
    assert sz["bitmap"] == (R * C + 7) // 8 and sz["scales"] == 2 * N * C


@pytest.mark.parametrize("args,status", [
    ((100, 128, 128, 128, 0), -2), ((128, 100, 128, 128, 0), -2), ((128, 128, 32, 128, 0), -2),
    ((128, 128, 128, 32, 0), -2), ((128, 128, 128, 128, 2), -1), ((128, 128, 128, 128, -1), -1)])
def test_packed_sizes_rejects(args, status):
    out = (ctypes.c_size_t * 7)()
    assert aq.lib().aq_packed_sizes(*args, out) == status


def _metadata(pmap):
    R, C = pmap.shape
    T = R * C
    bitmap = np.zeros((T + 7) // 8, np.uint8)
    off4 = np.zeros(R + 1, np.int32)
    off8 = np.zeros(R + 1, np.int32)
    idx = np.zeros(T, np.int32)
    t4 = ctypes.c_int32(-1)
    m = np.ascontiguousarray(pmap, dtype=np.uint8)
    rc = aq.lib().aq_pack_metadata(m.ctypes.data, R, C, bitmap.ctypes.data, off4.ctypes.data, off8.ctypes.data,
                                   idx.ctypes.data, ctypes.byref(t4))
    return rc, bitmap, off4, off8, idx, t4.value


@pytest.mark.parametrize("R,C,frac8,seed", [(1, 3, 0.34, 0), (3, 5, 0.5, 1), (8, 24, 0.25, 2), (40, 136, 0.3, 3),
                                            (7, 9, 0.0, 4), (7, 9, 1.0, 5)])
def test_pack_metadata_matches_oracle(R, C, frac8, seed):
    pmap = synth.precision_map(R, C, frac8, (seed,))
    rc, bitmap, off4, off8, idx, t4 = _metadata(pmap)
    assert rc == 0
    assert np.array_equal(bitmap, oracle.labels_to_bitmap(pmap))
    assert np.array_equal(off4, oracle.row_offsets(pmap, 4))
    assert np.array_equal(off8, oracle.row_offsets(pmap, 8))
    assert t4 == int(pmap.sum())
    for r in range(R):
        for j in range(C):
            assert idx[r * C + j] == oracle.physical_index(pmap, r, j, 4 if pmap[r, j] else 8)


def test_pack_metadata_worked_example_and_rejects_bad_label():
    rc, bitmap, off4, off8, idx, t4 = _metadata(np.array([[1, 0, 1]], np.uint8))
    assert rc == 0 and list(idx) == [0, 0, 1] and t4 == 2 and list(bitmap) == [5]
    rc, *_ = _metadata(np.array([[1, 2, 0]], np.uint8))
    assert rc == -1


def test_host_validation_rejects_before_any_launch():
    L = aq.lib()
    # activation quantization: bad M, K, ldx and alignment
    assert L.aq_quant_act(16, 0, 128, 128, 16, 16, None) == -1
    assert L.aq_quant_act(16, 1, 100, 128, 16, 16, None) == -1
    assert L.aq_quant_act(16, 1, 128, 64, 16, 16, None) == -1
    assert L.aq_quant_act(17, 1, 128, 128, 16, 16, None) == -1
    assert L.aq_quant_act(None, 1, 128, 128, 16, 16, None) == -1
    # linear calls: null struct, bad geometry, M out of range, bad dtype
    assert L.aq_linear_decode(None, 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    s = aq.AqPackedStruct(N=100, K=128, bN=128, bK=128, R=0, C=1, T4=0, T8=0)
    assert L.aq_linear_decode(ctypes.byref(s), 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -2
    s = aq.AqPackedStruct(N=128, K=128, bN=128, bK=128, R=1, C=1, T4=0, T8=1,
                          bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    assert L.aq_linear_decode(ctypes.byref(s), 16, 16, 65, None, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_decode(ctypes.byref(s), 16, 16, 1, None, 16, 7, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_prefill(ctypes.byref(s), 16, 16, 1, None, 16, 0, 64, 16, 1 << 20, None) == -1
    assert L.aq_linear_decode(ctypes.byref(s), 16, 16, 1, None, 16, 0, 128, None, 0, None) == -5
    assert L.aq_linear_prefill(ctypes.byref(s), 16, 16, 1, None, 16, 0, 128, 16, 8, None) == -5
    # token scales, bias and fp32 outputs are 4-byte words, bf16 outputs 2-byte words, the workspace 16-byte aligned
    assert L.aq_linear_decode(ctypes.byref(s), 16, 18, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_decode(ctypes.byref(s), 16, 16, 1, 18, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_prefill(ctypes.byref(s), 16, 16, 1, None, 18, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_prefill(ctypes.byref(s), 16, 16, 1, None, 17, 1, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_decode(ctypes.byref(s), 16, 16, 1, None, 16, 0, 128, 24, 1 << 20, None) == -1
    assert L.aq_linear_prefill(ctypes.byref(s), 16, 16, 1, None, 16, 0, 128, 24, 1 << 20, None) == -1
    assert L.aq_linear_decode_noalloc(ctypes.byref(s), 16, 18, 1, None, 16, 0, 128, None) == -1
    assert L.aq_linear_decode_noalloc(ctypes.byref(s), 16, 16, 1, None, 17, 1, 128, None) == -1
    assert L.aq_debug_tile_partials(ctypes.byref(s), 16, 1, 1, 18, 16, 1 << 20, None) == -1
    ws_args = [ctypes.pointer(s)]
    members = (ctypes.POINTER(aq.AqPackedStruct) * 1)(*ws_args)
    ys, lds = (ctypes.c_void_p * 1)(18), (ctypes.c_int * 1)(128)
    assert L.aq_linear_group(0, members, 1, 16, 128, 1, None, ys, lds, 0, 16, 1 << 20, None) == -1
    biases = (ctypes.c_void_p * 1)(18)
    ys[0] = 16
    assert L.aq_linear_group(0, members, 1, 16, 128, 1, biases, ys, lds, 0, 16, 1 << 20, None) == -1
    assert L.aq_linear_group(0, members, 1, 16, 128, 1, None, ys, lds, 0, 24, 1 << 20, None) == -1
    # packed buffers moved by bulk copies (w4, w8, scales) must be 16-byte aligned
    mis = aq.AqPackedStruct(N=128, K=128, bN=128, bK=128, R=1, C=1, T4=0, T8=1,
                            bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=18)
    assert L.aq_linear_prefill(ctypes.byref(mis), 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_decode(ctypes.byref(mis), 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    # weight quantizer: null, dtype, search flag, geometry, ldw and alignment
    qw = L.aq_quantize_weights
    assert qw(None, 0, 128, 128, 128, 128, 128, 16, 1, 16, 16, None) == -1
    assert qw(16, 2, 128, 128, 128, 128, 128, 16, 1, 16, 16, None) == -1
    assert qw(16, 0, 128, 128, 128, 128, 128, 16, 2, 16, 16, None) == -1
    assert qw(16, 0, 100, 128, 128, 128, 128, 16, 1, 16, 16, None) == -2
    assert qw(16, 0, 128, 128, 128, 128, 64, 16, 1, 16, 16, None) == -2
    assert qw(16, 0, 128, 128, 120, 128, 128, 16, 1, 16, 16, None) == -1
    assert qw(16, 0, 128, 128, 130, 128, 128, 16, 1, 16, 16, None) == -1
    assert qw(16, 1, 128, 128, 132, 128, 128, 16, 1, 16, 16, None) == -1
    assert qw(20, 0, 128, 128, 128, 128, 128, 16, 1, 16, 16, None) == -1
    assert qw(16, 0, 128, 128, 128, 128, 128, 16, 1, 24, 16, None) == -1
    assert qw(16, 0, 128, 128, 128, 128, 128, 16, 1, 16, 17, None) == -1   # fp16 scales are 2-byte words
    # scalar words: activation scales (4 B), the tile table (4 B), fp16 row scales into the packer (2 B)
    assert L.aq_quant_act(16, 1, 128, 128, 16, 18, None) == -1
    assert L.aq_quant_act_groups(16, 1, 128, 128, 16, 18, None) == -1
    odd_idx = aq.AqPackedStruct(N=128, K=128, bN=128, bK=128, R=1, C=1, T4=0, T8=1,
                                bitmap=16, row_off4=16, row_off8=16, tile_idx=18, w4=16, w8=16, scales=16)
    assert L.aq_linear_decode(ctypes.byref(odd_idx), 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_workspace_bytes(0, 1, ctypes.byref(odd_idx)) == 0
    pk_out = aq.AqPackedStruct(T4=0, bitmap=16, row_off4=16, row_off8=16, tile_idx=18, w4=16, w8=16, scales=16)
    assert L.aq_pack(16, 16, 16, 128, 128, 128, 128, ctypes.byref(pk_out), None) == -1
    pk_out.tile_idx = 16
    assert L.aq_pack(16, 17, 16, 128, 128, 128, 128, ctypes.byref(pk_out), None) == -1
    assert L.aq_workspace_bytes(0, 65, ctypes.byref(s)) == 0
    assert L.aq_workspace_bytes(0, 1, ctypes.byref(s)) >= 256
    assert L.aq_workspace_bytes(5, 1, ctypes.byref(s)) == 0
    assert L.aq_debug_tile_partials(ctypes.byref(s), 16, 1, 3, 16, 16, 1 << 20, None) == -1


def test_decode_workspace_sizes():
    """Up to 3 tokens the CUDA-core kernel needs only the status header; above,
    the tensor-core split-K partial sums grow with the token count."""
    L = aq.lib()
    s = aq.AqPackedStruct(N=1024, K=3072, bN=128, bK=128, R=8, C=24, T4=100, T8=92,
                          bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    b1 = L.aq_workspace_bytes(0, 1, ctypes.byref(s))
    b3 = L.aq_workspace_bytes(0, 3, ctypes.byref(s))
    b4 = L.aq_workspace_bytes(0, 4, ctypes.byref(s))
    b8 = L.aq_workspace_bytes(0, 8, ctypes.byref(s))
    b16 = L.aq_workspace_bytes(0, 16, ctypes.byref(s))
    b32 = L.aq_workspace_bytes(0, 32, ctypes.byref(s))
    assert b1 == b3 == 256
    assert b32 > b16 > b8 > b4 > 256


def test_group_workspace_sizes():
    L = aq.lib()
    P = ctypes.POINTER(aq.AqPackedStruct)
    mk = lambda N: aq.AqPackedStruct(N=N, K=3072, bN=128, bK=128, R=N // 128, C=24, T4=0, T8=(N // 128) * 24,
                                     bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    q, k, v = mk(3072), mk(1024), mk(1024)
    arr = (P * 3)(ctypes.pointer(q), ctypes.pointer(k), ctypes.pointer(v))
    assert L.aq_group_workspace_bytes(0, 1, arr, 3) == 256          # fused: one launch, no scratch
    assert L.aq_group_workspace_bytes(0, 16, arr, 3) >= 16 * 3072   # quantized input kept in the workspace
    assert L.aq_group_workspace_bytes(1, 300, arr, 3) >= 300 * 3072
    assert L.aq_group_workspace_bytes(0, 65, arr, 3) == 0
    assert L.aq_group_workspace_bytes(0, 1, arr, 4) == 0
    bad = mk(1024)
    bad.K, bad.C = 2048, 16
    arr2 = (P * 2)(ctypes.pointer(q), ctypes.pointer(bad))
    assert L.aq_group_workspace_bytes(0, 1, arr2, 2) == 0


def test_paper_accounting_reproduces_table16():
    # App. H.3.3 Table 16 packed bits per weight for the Llama-3.2-3B shapes at
    # 64 x 64 tiles, model-wide W4 count round(rho |T|) filled projection by
    # projection, through the library's eq. 18 accounting
    import json, os
    with open(os.path.join(os.path.dirname(__file__), "golden", "table16_packed_bpw.json")) as f:
        g = json.load(f)
    bN, bK = g["tile"]
    shapes = synth.projections("llama-3.2-3b") * synth.MODELS["llama-3.2-3b"]["layers"]
    tiles = [(n // bN) * (k // bK) for _, n, k in shapes]
    for rho, want in zip(g["w4_fraction"], g["packed_bpw_2dp"]):
        left, S, W = int(round(rho * sum(tiles))), 0, 0
        for (_, n, k), t in zip(shapes, tiles):
            t4 = min(left, t)
            left -= t4
            S += aq.aq_paper_packed_bytes(n // bN, k // bK, t4, bN, bK)
            W += n * k
        assert round(8 * S / W, 2) == pytest.approx(want, abs=1e-9), rho


@pytest.mark.parametrize("R,C,T4,bN,bK", [(1, 1, 0, 2, 2), (3, 5, 7, 64, 64), (40, 24, 960, 128, 128),
                                          (17, 9, 0, 64, 128), (2, 3, 6, 1, 2)])
def test_paper_accounting_matches_oracle_and_rejects(R, C, T4, bN, bK):
    assert aq.aq_paper_packed_bytes(R, C, T4, bN, bK) == oracle.paper_packed_bytes(R, C, T4, bN, bK)
    L, out = aq.lib(), ctypes.c_size_t()
    assert L.aq_paper_packed_bytes(R, C, R * C + 1, bN, bK, ctypes.byref(out)) == -1
    assert L.aq_paper_packed_bytes(R, C, -1, bN, bK, ctypes.byref(out)) == -1
    assert L.aq_paper_packed_bytes(R, C, T4, 3, 3, ctypes.byref(out)) == -1
    assert L.aq_paper_packed_bytes(0, C, 0, bN, bK, ctypes.byref(out)) == -1
    assert L.aq_paper_packed_bytes(R, C, T4, bN, bK, None) == -1


def test_long_prefill_sizes_and_validation():
    L = aq.lib()
    s = aq.AqPackedStruct(N=256, K=384, bN=128, bK=128, R=2, C=3, T4=2, T8=4,
                          bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    a256 = lambda b: (b + 255) // 256 * 256
    want = a256(6 * 128 * 128) + a256(4 * 6) + 2 * a256(4 * 3) + a256(1)
    assert L.aq_expanded_bytes(ctypes.byref(s)) == want
    bad = aq.AqPackedStruct(N=100, K=384, bN=128, bK=128, R=0, C=3, T4=0, T8=0)
    assert L.aq_expanded_bytes(ctypes.byref(bad)) == 0
    out = aq.AqPackedStruct()
    assert L.aq_expand_int8(ctypes.byref(s), None, want, ctypes.byref(out), None) == -1
    assert L.aq_expand_int8(ctypes.byref(s), 4096 + 16, want, ctypes.byref(out), None) == -1  # not 256-byte aligned
    assert L.aq_expand_int8(ctypes.byref(s), 4096, want - 1, ctypes.byref(out), None) == -5
    assert L.aq_expand_int8(ctypes.byref(bad), 4096, want, ctypes.byref(out), None) == -2
    ws = L.aq_workspace_bytes(1, 300, ctypes.byref(s))
    f = L.aq_linear_prefill_expanded
    assert f(ctypes.byref(s), 16, 16, 300, None, 16, 0, 256, 16, ws, None, want, None) == -1
    assert f(ctypes.byref(s), 16, 16, 300, None, 16, 0, 256, 16, ws, 4096, want - 1, None) == -5
    assert f(ctypes.byref(s), 16, 16, 300, None, 16, 0, 256, 16, ws - 1, 4096, want, None) == -5


def test_paper_form_activation_quantizer_validation():
    L = aq.lib()
    assert L.aq_act_group_rows(1) == 1 and L.aq_act_group_rows(2) == 16 and L.aq_act_group_rows(0) == 0
    f = L.aq_quant_act_groups
    assert f(None, 1, 128, 128, 16, 16, None) == -1
    assert f(16, 0, 128, 128, 16, 16, None) == -1
    assert f(16, 1, 96, 96, 16, 16, None) == -1       # K not a multiple of 64
    assert f(16, 1, 128, 120, 16, 16, None) == -1     # ldx < K
    assert f(16, 1, 128, 132, 16, 16, None) == -1     # ldx not a multiple of 8
    assert f(24, 1, 128, 128, 16, 16, None) == -1     # x not 16-byte aligned
    assert f(16, 1, 128, 128, 20, 16, None) == -1     # xq not 8-byte aligned


def test_paper_exact_mode_validation():
    """The paper-exact entries (bK = 64, per-tile fp32 scales) and the per-token
    layer reject each other's packed structs, before any launch."""
    L = aq.lib()
    sizes = aq.aq_packed_sizes(128, 128, 64, 64, 1)
    assert sizes["w8"] == 3 * 64 * 64 and sizes["w4"] == 64 * 32 and sizes["scales"] >= 4 * 4
    assert L.aq_pack_tiles(None, 16, 16, 128, 128, 64, 64, None, None) == -1
    out = aq.AqPackedStruct()
    assert L.aq_pack_tiles(16, 16, 16, 128, 128, 64, 128, ctypes.byref(out), None) == -2  # bK must be 64
    assert L.aq_pack_tiles(16, 16, 16, 128, 96, 64, 64, ctypes.byref(out), None) == -2    # K % 64
    assert L.aq_pack(16, 16, 16, 128, 128, 64, 64, ctypes.byref(out), None) == -2         # per-row form: bK = 128
    bufs = dict(bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    paper = aq.AqPackedStruct(N=128, K=128, bN=64, bK=64, R=2, C=2, T4=0, T8=4, scale_kind=aq.AQ_SCALES_TILE_FP32,
                              **bufs)
    rowform = aq.AqPackedStruct(N=128, K=128, bN=128, bK=128, R=1, C=1, T4=0, T8=1, **bufs)
    lin = L.aq_paper_linear
    assert lin(ctypes.byref(rowform), 16, 16, 1, None, None, 16, 128, None) == -1   # fp16 row-scale struct
    wrong_kind = aq.AqPackedStruct(N=128, K=128, bN=64, bK=64, R=2, C=2, T4=0, T8=4, **bufs)
    assert lin(ctypes.byref(wrong_kind), 16, 16, 1, None, None, 16, 128, None) == -1
    bad_geo = aq.AqPackedStruct(N=128, K=128, bN=128, bK=128, R=1, C=1, T4=0, T8=1,
                                scale_kind=aq.AQ_SCALES_TILE_FP32, **bufs)
    assert lin(ctypes.byref(bad_geo), 16, 16, 1, None, None, 16, 128, None) == -2
    assert lin(ctypes.byref(paper), 16, 16, 0, None, None, 16, 128, None) == -1      # M < 1
    assert lin(ctypes.byref(paper), 16, 16, 65536 * 16, None, None, 16, 128, None) == -1  # > 65535 row groups
    assert lin(ctypes.byref(paper), 16, 16, 1, None, None, None, 128, None) == -1    # no output
    assert lin(ctypes.byref(paper), 16, 16, 1, None, None, 16, 100, None) == -1      # ldy < N
    assert lin(ctypes.byref(paper), 24, 16, 1, None, None, 16, 128, None) == -1      # xq not 16-byte aligned
    assert lin(ctypes.byref(paper), 16, 18, 1, None, None, 16, 128, None) == -1      # sx not 4-byte aligned
    assert lin(ctypes.byref(paper), 16, 16, 1, 18, None, 16, 128, None) == -1        # u
    assert lin(ctypes.byref(paper), 16, 16, 1, None, 18, 16, 128, None) == -1        # bias
    assert lin(ctypes.byref(paper), 16, 16, 1, None, None, 18, 128, None) == -1      # y
    assert L.aq_debug_paper_partials(ctypes.byref(paper), 16, 1, None, None) == -1
    paper_odd_idx = aq.AqPackedStruct(N=128, K=128, bN=64, bK=64, R=2, C=2, T4=0, T8=4,
                                      scale_kind=aq.AQ_SCALES_TILE_FP32, **dict(bufs, tile_idx=18))
    assert lin(ctypes.byref(paper_odd_idx), 16, 16, 1, None, None, 16, 128, None) == -1
    paper_out = aq.AqPackedStruct(T4=0, **bufs)
    assert L.aq_pack_tiles(16, 18, 16, 128, 128, 64, 64, ctypes.byref(paper_out), None) == -1  # fp32 tile scales
    assert L.aq_debug_paper_partials(ctypes.byref(paper), 16, 1, 18, None) == -1    # P not 4-byte aligned
    # the per-token layer refuses a paper-form struct
    paper128 = aq.AqPackedStruct(N=128, K=128, bN=128, bK=128, R=1, C=1, T4=0, T8=1,
                                 scale_kind=aq.AQ_SCALES_TILE_FP32, **bufs)
    assert L.aq_linear_decode(ctypes.byref(paper128), 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_linear_prefill(ctypes.byref(paper128), 16, 16, 1, None, 16, 0, 128, 16, 1 << 20, None) == -1
    assert L.aq_workspace_bytes(0, 1, ctypes.byref(paper128)) == 0
    q = L.aq_paper_quant_act
    assert q(None, 1, 128, 128, None, 16, 16, None) == -1
    assert q(16, 0, 128, 128, None, 16, 16, None) == -1
    assert q(16, 1, 96, 96, None, 16, 16, None) == -1      # K % 64
    assert q(16, 1, 128, 120, None, 16, 16, None) == -1    # ldx < K
    assert q(16, 1, 128, 128, 24, 16, 16, None) == -1      # V staged with 16-byte loads
    assert q(17, 1, 128, 128, None, 16, 16, None) == -1    # x read as 2-byte words
    assert q(16, 1, 128, 128, None, 16, 18, None) == -1    # sx written as 4-byte words


def _split_count(M, N, K, sms=148):
    """Splits of the tensor-core decode plan (a restatement of the rule for this test)."""
    C, blocks = K // 128, -(-N // 128)
    per = 5 if M <= 16 else 8 if M <= 32 else 20
    s = max(1, min(min(C // per, 8), sms // blocks))
    return 1 if (M >= 32 and 3 * blocks >= sms) else s


@pytest.mark.parametrize("M,N,K", [(16, 3072, 3072), (32, 3072, 3072), (64, 3072, 3072), (64, 3072, 8192),
                                   (32, 8192, 3072), (16, 4096, 14336), (4, 1024, 3072), (64, 4096, 14336)])
def test_decode_split_plan_in_workspace_sizes(M, N, K):
    """The workspace of a tensor-core decode call holds the header, one split
    counter per 128-row block and, with splits, S partial-sum planes of
    N x (M rounded up to 4) floats: at least 5 / 8 / 20 input tiles per split at
    <= 16 / <= 32 / <= 64 tokens, one wave, at most 8, and no split from 32
    tokens when the row blocks fill a third of the GPU."""
    L = aq.lib()
    R, C = N // 128, K // 128
    s = aq.AqPackedStruct(N=N, K=K, bN=128, bK=128, R=R, C=C, T4=R * C, T8=0,
                          bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    counters = (R * 4 + 255) // 256 * 256
    S = _split_count(M, N, K)
    want = 256 + counters + (S * ((M + 3) // 4 * 4) * N * 4 if S > 1 else 0)
    assert L.aq_workspace_bytes(0, M, ctypes.byref(s)) == want


def test_group_workspace_covers_the_grouped_tensor_core_launch():
    """A decode group whose members are whole 128-row blocks runs as one
    tensor-core launch over all their rows: its workspace holds that launch's
    partial sums (split plan over the summed row blocks) before the prepared
    activations."""
    L = aq.lib()
    P = ctypes.POINTER(aq.AqPackedStruct)
    mk = lambda N: aq.AqPackedStruct(N=N, K=8192, bN=128, bK=128, R=N // 128, C=64, T4=0, T8=(N // 128) * 64,
                                     bitmap=16, row_off4=16, row_off8=16, tile_idx=16, w4=16, w8=16, scales=16)
    members = [mk(1024), mk(256), mk(256)]
    arr = (P * 3)(*[ctypes.pointer(m) for m in members])
    M, N = 16, 1536
    S = _split_count(M, N, 8192)
    blocks = N // 128
    lin = 256 + (blocks * 4 + 255) // 256 * 256 + S * M * N * 4
    align = lambda b: (b + 255) // 256 * 256
    assert L.aq_group_workspace_bytes(0, M, arr, 3) >= align(lin) + align(M * 8192) + align(M * 4)
