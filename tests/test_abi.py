"""The C-ABI library loads, exports every entry point include/*.h declares, and rejects
invalid arguments on the host before anything is enqueued (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

from tests.conftest import ROOT

import trellis_quantized_moe_gemv_b200.build as tqbuild


@pytest.fixture(scope="module")
def lib():
    tqbuild.build()
    from trellis_quantized_moe_gemv_b200 import api
    return api.lib()


def declared_functions():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(path).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w]*\s*\**\s*\**\s*([A-Za-z_]\w*)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("trellis_decode", "hadamard128", "trellis_gemv", "route_topk", "route_permute",
                     "route_unpermute", "moe_trellis_gemv", "moe_trellis_gemm",
                     "moe_trellis_workspace_size", "tq_status_string", "tq_abi_version",
                     "tq_device_status", "trellis_encode", "trellis_encode_workspace_size",
                     "route_gather_rows", "route_topk_permute"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_status_strings(lib):
    from trellis_quantized_moe_gemv_b200 import api
    assert api.abi_version() == 3
    for code in range(7):
        assert lib.tq_status_string(code)
    assert b"ALIGNMENT" in lib.tq_status_string(3)
    assert lib.tq_status_string(99) == b"unknown tq_status"


FAKE = ctypes.c_void_p(0x10000)        # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10004)


def test_host_validation_rejects_bad_arguments(lib):
    # widths, shapes
    assert lib.trellis_decode(FAKE, 5, 16, 16, FAKE, None) == 1
    assert lib.trellis_decode(FAKE, 2, 15, 16, FAKE, None) == 1
    assert lib.trellis_decode(None, 2, 16, 16, FAKE, None) == 1
    assert lib.trellis_decode(MISALIGNED, 2, 16, 16, FAKE, None) == 3
    assert lib.trellis_decode(FAKE, 2, 0, 16, FAKE, None) == 0          # empty: no-op
    assert lib.trellis_decode_e4m3(FAKE, 5, 16, 16, FAKE, None) == 1
    assert lib.trellis_decode_e4m3(FAKE, 2, 16, 24, FAKE, None) == 1
    assert lib.trellis_decode_e4m3(MISALIGNED, 2, 16, 16, FAKE, None) == 3
    assert lib.trellis_decode_e4m3(FAKE, 2, 0, 16, FAKE, None) == 0
    assert lib.hadamard128(FAKE, 0, 4, 100, FAKE, None) == 1            # cols % 128
    assert lib.hadamard128(FAKE, 7, 4, 128, FAKE, None) == 1            # dtype
    assert lib.hadamard128(MISALIGNED, 0, 4, 128, FAKE, None) == 3
    assert lib.hadamard128(FAKE, 0, 0, 128, FAKE, None) == 0
    big = ctypes.c_size_t(1 << 40)
    assert lib.trellis_gemv(FAKE, FAKE, 2, 16, 64, FAKE, 1, FAKE, FAKE, big, None) == 1   # cols % 128
    assert lib.trellis_gemv(FAKE, FAKE, 1, 16, 128, FAKE, 1, FAKE, FAKE, big, None) == 1  # K
    assert lib.trellis_gemv(FAKE, FAKE, 2, 16, 32768, FAKE, 1, FAKE, FAKE, big, None) == 2  # cols
    assert lib.trellis_gemv(FAKE, FAKE, 2, 16, 128, FAKE, 70000, FAKE, FAKE, big, None) == 2
    assert lib.trellis_gemv(FAKE, FAKE, 2, 16, 128, FAKE, 0, FAKE, None, 0, None) == 0
    # workspace: quantised rows (four half-word planes: the main word and the residual
    # word, high and low bytes), 16 bytes of metadata per row, 16 bytes per output
    need = lib.trellis_gemv_workspace_size(32, 256, 3)
    assert need == 3 * 4 * 256 * 2 + 256 + 32 * 3 * 16
    assert lib.trellis_gemv(FAKE, FAKE, 2, 32, 256, FAKE, 3, FAKE, FAKE, ctypes.c_size_t(need - 1),
                            None) == 4
    assert lib.trellis_gemv(FAKE, FAKE, 2, 32, 256, FAKE, 3, FAKE, MISALIGNED, ctypes.c_size_t(need),
                            None) == 3
    assert lib.route_topk(FAKE, 4, 384, 0, FAKE, FAKE, None) == 1
    assert lib.route_topk(FAKE, 4, 4, 8, FAKE, FAKE, None) == 1         # k > E
    assert lib.route_topk(FAKE, 0, 384, 8, FAKE, FAKE, None) == 0
    assert lib.route_permute(FAKE, 4, 8, 2000, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib.route_unpermute(FAKE, FAKE, FAKE, 4, 8, 6, FAKE, None) == 1
    assert lib.route_unpermute(MISALIGNED, FAKE, FAKE, 4, 8, 8, FAKE, None) == 3
    # route_topk_permute(logits, T, E, k, ids, w, counts, offsets, perm, inv, active, n_active, stream)
    assert lib.route_topk_permute(FAKE, 4, 384, 0, *[FAKE] * 8, None) == 1          # k
    assert lib.route_topk_permute(FAKE, 4, 2000, 8, *[FAKE] * 8, None) == 1         # E
    assert lib.route_topk_permute(FAKE, 4, 384, 8, FAKE, FAKE, None, *[FAKE] * 5, None) == 1
    # route_gather_rows(src, dtype, src_rows, cols, index, divisor, rows, out, stream)
    assert lib.route_gather_rows(FAKE, 3, 4, 8, FAKE, 1, 4, FAKE, None) == 1         # dtype
    assert lib.route_gather_rows(FAKE, 0, 4, 4, FAKE, 1, 4, FAKE, None) == 1         # 8-byte rows
    assert lib.route_gather_rows(FAKE, 2, 4, 4, FAKE, 0, 4, FAKE, None) == 1         # divisor
    assert lib.route_gather_rows(FAKE, 2, 4, 4, None, 1, 4, FAKE, None) == 1
    assert lib.route_gather_rows(MISALIGNED, 2, 4, 4, FAKE, 1, 4, FAKE, None) == 3
    assert lib.route_gather_rows(FAKE, 1, 4, 8, FAKE, 1, 0, FAKE, None) == 0         # empty: no-op


def _layer_struct(K=2, E=16, D=256, F=128, n_groups=1):
    from trellis_quantized_moe_gemv_b200 import api
    st = api.TqMoeLayer()
    st.E, st.D, st.F, st.n_groups = E, D, F, n_groups
    for g in range(n_groups):
        w = st.groups[g]
        w.K, w.n_experts = K, E
        for key in ("expert_ids", "gate", "up", "down", "s_gate", "s_up", "s_down"):
            setattr(w, key, 0x10000)
    st.expert_slot = 0x10000
    return st


def test_moe_workspace_and_layer_validation(lib):
    st = _layer_struct()
    need = lib.moe_trellis_workspace_size(ctypes.byref(st), 16, 8)
    # GEMV: per-route gate and up results (fp32; this layer's 16 experts x 2 items get 2
    # column splits: min(8, ceil(3 * SMs / 32), D / 128)), h' and x' as fixed point (four
    # half-word planes per value: main and residual word) and 16 bytes of metadata per row
    gemv_need = 128 * 2 * 2 * 128 * 4 + 128 * 4 * 128 * 2 + 128 * 16 + 16 * 4 * 256 * 2 + 256
    gemv_need += 256     # the fused kernel's work queue and per-expert counters: (1 + 2E) ints
    # the GEMM path also holds route-ordered activations (fp16), their row sums, h, h',
    # its row sums and power-of-two row scales, and the tile list
    gemm_need = 128 * 256 * 2 + 512 + 128 * 128 * 4 + 128 * 128 * 2 + 512 + 512 + 256
    assert need == max(gemv_need, gemm_need)
    bad = _layer_struct(K=5)
    assert lib.moe_trellis_workspace_size(ctypes.byref(bad), 16, 8) == 0
    bad = _layer_struct(D=200)
    assert lib.moe_trellis_workspace_size(ctypes.byref(bad), 16, 8) == 0
    bad = _layer_struct()
    bad.codebook = 7                                      # unknown codebook
    assert lib.moe_trellis_workspace_size(ctypes.byref(bad), 16, 8) == 0
    fp8 = _layer_struct()
    fp8.codebook = 1                                      # pair trellis: GEMM only
    assert lib.moe_trellis_workspace_size(ctypes.byref(fp8), 16, 8) == need
    assert lib.moe_trellis_gemv(ctypes.byref(fp8), *[FAKE] * 5, 16, 8, FAKE, FAKE, need, None) == 2
    assert lib.moe_trellis_gemv_noalloc(ctypes.byref(fp8), *[FAKE] * 5, 1, 8, FAKE, None) == 2
    args = [FAKE] * 5
    # workspace too small
    assert lib.moe_trellis_gemv(ctypes.byref(st), *args, 16, 8, FAKE, FAKE, gemv_need - 1, None) == 4
    assert lib.moe_trellis_gemm(ctypes.byref(st), *args, 16, 8, FAKE, FAKE, gemm_need - 1, None) == 4
    assert lib.moe_trellis_gemv(ctypes.byref(st), *args, 16, 8, FAKE, None, need, None) == 4
    # misaligned activations
    assert lib.moe_trellis_gemv(ctypes.byref(st), MISALIGNED, *args[1:], 16, 8, FAKE, FAKE, need,
                                None) == 3
    # T = 0 is a no-op
    assert lib.moe_trellis_gemv(ctypes.byref(st), *args, 0, 8, FAKE, FAKE, 0, None) == 0
    # misaligned bit streams
    mis = _layer_struct()
    mis.groups[0].gate = 0x10004
    assert lib.moe_trellis_gemv(ctypes.byref(mis), *args, 16, 8, FAKE, FAKE, need, None) == 3
    # layer sign vectors of the two-sided transform: all four or none, 4-byte aligned
    part = _layer_struct()
    part.sign_x = part.sign_gu = 0x10000
    assert lib.moe_trellis_workspace_size(ctypes.byref(part), 16, 8) == 0
    assert lib.moe_trellis_gemv(ctypes.byref(part), *args, 16, 8, FAKE, FAKE, need, None) == 1
    signed = _layer_struct()
    signed.sign_x = signed.sign_gu = signed.sign_h = signed.sign_y = 0x10000
    need2 = lib.moe_trellis_workspace_size(ctypes.byref(signed), 16, 8)
    assert need2 >= need
    signed.sign_h = 0x10002
    assert lib.moe_trellis_gemv(ctypes.byref(signed), *args, 16, 8, FAKE, FAKE, need2, None) == 3
    assert lib.hadamard128_signed(FAKE, 0, 4, 128, None, FAKE, None) == 1
    assert lib.route_unpermute_signed(FAKE, FAKE, FAKE, 4, 8, 200, FAKE, FAKE, None) == 1


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    from trellis_quantized_moe_gemv_b200 import api
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(api.TQError):
        api.lib()


def test_encode_validation(lib):
    # workspace: 255 backpointer rows of 2^(16-K) bytes per resident CTA (one per tile here)
    assert lib.trellis_encode_workspace_size(2, 32, 32) == 4 * 255 * (1 << 14)
    assert lib.trellis_encode_workspace_size(4, 16, 16) == 255 * (1 << 12)
    assert lib.trellis_encode_workspace_size(5, 16, 16) == 0
    assert lib.trellis_encode_workspace_size(2, 20, 16) == 0
    assert lib.trellis_encode_workspace_size(3, 0, 16) == 0
    need = lib.trellis_encode_workspace_size(3, 32, 32)
    assert lib.trellis_encode(FAKE, 5, 32, 32, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.trellis_encode(FAKE, 3, 30, 32, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.trellis_encode(FAKE, 3, 32, 32, FAKE, FAKE, FAKE, need - 1, None) == 4
    assert lib.trellis_encode(FAKE, 3, 32, 32, FAKE, None, MISALIGNED, need, None) == 3
    assert lib.trellis_encode(None, 3, 32, 32, FAKE, None, FAKE, need, None) == 1
    assert lib.trellis_encode(None, 3, 0, 32, None, None, None, 0, None) == 0   # no tiles: no-op
