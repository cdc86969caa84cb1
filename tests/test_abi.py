"""The C ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a device (no GPU needed)."""
import ctypes
import os
import re

import pytest

from quantized_lora_fine_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*([a-z][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_the_five_operations():
    names = declared_functions()
    for op in ("nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd", "nf4_layer_error_rank"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(_lib.SIGNATURES), set(names) - set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert lib.qlora_status_str(0) == b"ok"
    assert b"time" in lib.qlora_status_str(9)


def test_workspace_sizes_are_host_only(lib):
    assert lib.qlora_fwd_workspace_size(8192, 4096, 4096, 16) > 4096 * 64 * 4
    assert lib.qlora_bwd_workspace_size(8192, 4096, 4096, 16) > 0
    assert lib.qlora_fwd_workspace_size(0, 4096, 4096, 16) == 0
    n = (ctypes.c_int64 * 2)(4096 * 4096, 11008 * 4096)
    assert lib.nf4_layer_error_rank_workspace_size(2, n) > 0


def test_host_validation_before_any_launch(lib):
    q = _lib.NF4QConfig(64, 0, 256)
    # NULL weight pointer
    assert lib.nf4_quantize(None, 0, 64, 64, q, None, None, None, None, None, 0, None) == 1
    # bad dtype
    assert lib.nf4_quantize(None, 7, 64, 64, q, None, None, None, None, None, 0, None) == 4
    # unsupported blocksize
    assert lib.nf4_quantize(None, 0, 64, 64, _lib.NF4QConfig(32, 0, 256), None, None, None, None, None, 0, None) == 5
    # linear: bad shapes are refused on the host
    w = _lib.QLoraWeight()
    w.out, w.in_ = 4096, 1000
    w.q = q
    assert lib.qlora_linear_fwd(ctypes.byref(w), None, 8, None, None, 16, 2.0, None, None, None, 0, None) == 2
    w.in_ = 4096
    assert lib.qlora_linear_fwd(ctypes.byref(w), None, 8, None, None, 12, 2.0, None, None, None, 0, None) == 2
    # missing codes
    assert lib.qlora_linear_fwd(ctypes.byref(w), None, 8, None, None, 16, 2.0, None, None, None, 0, None) == 1
    # misaligned weight pointer
    w.codes = 0x1001
    w.absmax = 0x2000
    assert lib.qlora_linear_fwd(ctypes.byref(w), None, 8, None, None, 16, 2.0, None, None, None, 0, None) == 3
    # layer error: K out of range, numel not a multiple of 64
    ptrs = (ctypes.c_void_p * 1)(0x1000)
    n = (ctypes.c_int64 * 1)(100)
    assert lib.nf4_layer_error_rank(1, ptrs, n, 0, q, 2, None, None, None, None, 0, None) == 2
    assert lib.nf4_layer_error_rank(1, ptrs, n, 0, q, 1, 0x10, 0x10, 0x10, None, 0, None) == 2
    # batch quantize: n out of range, odd element count, misaligned codes, missing absmax
    cp = (ctypes.c_void_p * 1)(0x2000)
    am = (ctypes.c_void_p * 1)(0x3000)
    none = (ctypes.c_void_p * 1)(0)
    assert lib.nf4_quantize_batch(0, ptrs, n, 0, q, cp, am, none, none, 0x4000, 256, None) == 2
    n_odd = (ctypes.c_int64 * 1)(101)
    assert lib.nf4_quantize_batch(1, ptrs, n_odd, 0, q, cp, am, none, none, 0x4000, 256, None) == 2
    cp_bad = (ctypes.c_void_p * 1)(0x2001)
    assert lib.nf4_quantize_batch(1, ptrs, n, 0, q, cp_bad, am, none, none, 0x4000, 256, None) == 3
    assert lib.nf4_quantize_batch(1, ptrs, n, 0, q, cp, none, none, none, 0x4000, 256, None) == 1
    # two-part forward: bad rank; the misaligned weight above
    assert lib.qlora_lora_down(None, 8, 4096, None, 12, None, None, 0, None) == 2
    assert lib.qlora_linear_fwd_t(ctypes.byref(w), 0x1000, 8, None, 0x1000, 16, 2.0, 0x1000, None, 0, None) == 3

    # merge: in not a multiple of 64, rank out of range, misaligned codes / output, short workspace
    m = _lib.QLoraWeight()
    m.out, m.in_, m.q = 128, 100, q
    m.codes, m.absmax = 0x2000, 0x3000
    assert lib.qlora_lora_merge(ctypes.byref(m), 0x1000, 0x1000, 8, 2.0, 0x4000, None) == 2
    m.in_ = 128
    assert lib.qlora_lora_merge(ctypes.byref(m), 0x1000, 0x1000, 0, 2.0, 0x4000, None) == 2
    assert lib.qlora_lora_merge(ctypes.byref(m), None, 0x1000, 8, 2.0, 0x4000, None) == 1
    assert lib.qlora_lora_merge(ctypes.byref(m), 0x1000, 0x1000, 8, 2.0, 0x4001, None) == 3
    m.codes = 0x2001
    assert lib.qlora_lora_merge(ctypes.byref(m), 0x1000, 0x1000, 8, 2.0, 0x4000, None) == 3
    m.codes = 0x2000
    need = lib.qlora_lora_merge_requantize_workspace_size(128, 128)
    assert need >= 128 * 2 * 4          # the fp32 scales (status word in front)
    assert lib.qlora_lora_merge_requantize_workspace_size(0, 128) == 0
    assert lib.qlora_lora_merge_requantize(ctypes.byref(m), 0x1000, 0x1000, 8, 2.0, q, 0x5000, 0x6000, None, None,
                                           0x7000, need - 1, None) == 7
    assert lib.qlora_lora_merge_requantize(ctypes.byref(m), 0x1000, 0x1000, 8, 2.0, q, 0x5000, None, None, None,
                                           0x7000, need, None) == 1

def test_product_path_refuses_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError):
        _lib.load(str(tmp_path / "missing.so"))


def test_k_from_fraction_is_round_half_up(lib):
    """The host-only fraction rule agrees with the oracle's exact rational rule
    (0.2 of 144 keeps 29) and rejects bad fractions."""
    from fractions import Fraction
    from oracle import layer_error
    k = ctypes.c_int32(0)
    assert lib.nf4_k_from_fraction(1, 5, 144, ctypes.byref(k)) == 0 and k.value == 29
    assert lib.nf4_k_from_fraction(7, 20, 10, ctypes.byref(k)) == 0 and k.value == 4      # 3.5 rounds up
    import random
    rnd = random.Random(1)
    for _ in range(2000):
        den = rnd.randint(1, 10 ** 6)
        num = rnd.randint(0, den)
        L = rnd.randint(0, 5000)
        assert lib.nf4_k_from_fraction(num, den, L, ctypes.byref(k)) == 0
        assert k.value == layer_error.k_from_budget(Fraction(num, den), L), (num, den, L)
    assert lib.nf4_k_from_fraction(1, 0, 10, ctypes.byref(k)) == 2
    assert lib.nf4_k_from_fraction(3, 2, 10, ctypes.byref(k)) == 2
    assert lib.nf4_k_from_fraction(1, 2, 10, None) == 1
    # budget rule: negative budget, missing K output
    q = _lib.NF4QConfig(64, 0, 256)
    ptrs = (ctypes.c_void_p * 1)(0x1000)
    n = (ctypes.c_int64 * 1)(4096)
    assert lib.nf4_layer_error_rank_budget(1, ptrs, n, 0, q, -1, 0x10, 0x10, 0x10, 0x10, 0x2000, 1 << 20, None) == 2
    assert lib.nf4_layer_error_rank_budget(1, ptrs, n, 0, q, 100, 0x10, 0x10, 0x10, None, 0x2000, 1 << 20, None) == 1


def test_empty_inputs_are_refused_on_the_host(lib):
    """Empty inputs (no rows, no columns, no tokens, no layers, rank 0) return
    QLORA_ERR_SHAPE before any device work; workspace sizes for them are 0."""
    q = _lib.NF4QConfig(64, 0, 256)
    for out, inp in ((0, 64), (64, 0), (0, 0)):
        assert lib.nf4_quantize(0x1000, 0, out, inp, q, 0x2000, 0x3000, None, None, 0x4000, 256, None) == 2
    w = _lib.QLoraWeight()
    w.out, w.in_, w.q = 256, 256, q
    w.codes, w.absmax = 0x2000, 0x3000
    assert lib.qlora_linear_fwd(ctypes.byref(w), 0x1000, 0, 0x1000, 0x1000, 16, 2.0, 0x1000, None, 0x4000,
                                1 << 20, None) == 2
    assert lib.qlora_linear_bwd(ctypes.byref(w), 0x1000, 0x1000, 0, 0x1000, 0x1000, 16, 2.0, 0x1000, 0x1000,
                                0x1000, 0x1000, 0x4000, 1 << 20, None) == 2
    assert lib.qlora_fwd_workspace_size(0, 256, 256, 16) == 0
    assert lib.qlora_bwd_workspace_size(0, 256, 256, 16) == 0
    ptrs = (ctypes.c_void_p * 1)(0x1000)
    n = (ctypes.c_int64 * 1)(0)
    assert lib.nf4_layer_error_rank(0, ptrs, n, 0, q, 0, 0x10, 0x10, 0x10, 0x2000, 1 << 20, None) == 2
    assert lib.nf4_layer_error_rank(1, ptrs, n, 0, q, 0, 0x10, 0x10, 0x10, 0x2000, 1 << 20, None) == 2
    m = _lib.QLoraWeight()
    m.out, m.in_, m.q = 0, 64, q
    m.codes, m.absmax = 0x2000, 0x3000
    assert lib.qlora_lora_merge(ctypes.byref(m), 0x1000, 0x1000, 8, 2.0, 0x4000, None) == 2
    assert lib.qlora_lora_merge_requantize_workspace_size(0, 64) == 0


def test_residual_stage_host_validation(lib):
    q = _lib.NF4QConfig(64, 0, 256)
    w1 = _lib.QLoraWeight()
    w1.out, w1.in_, w1.q = 128, 64, q
    w1.codes, w1.absmax = 0x2000, 0x3000
    need = lib.nf4_quantize_residual_workspace_size(128 * 64)
    assert need >= 128 * 64 * 4
    assert lib.nf4_quantize_residual(0x1000, ctypes.byref(w1), q, 0x5000, 0x6000, None, None, 0x7000, need - 1,
                                     None) == 7
    assert lib.nf4_quantize_residual(0x1001, ctypes.byref(w1), q, 0x5000, 0x6000, None, None, 0x7000, need,
                                     None) == 3
    assert lib.nf4_quantize_residual(None, ctypes.byref(w1), q, 0x5000, 0x6000, None, None, 0x7000, need, None) == 1
    w1.is_bf16 = 1
    assert lib.nf4_quantize_residual(0x1000, ctypes.byref(w1), q, 0x5000, 0x6000, None, None, 0x7000, need,
                                     None) == 5
    w1.is_bf16 = 0
    w2 = _lib.QLoraWeight()
    w2.out, w2.in_, w2.q = 64, 128, q
    w2.codes, w2.absmax = 0x2000, 0x3000
    assert lib.nf4_dequantize_two_stage(ctypes.byref(w1), ctypes.byref(w2), 0x8000, None) == 2
    w1.in_ = 63
    assert lib.nf4_dequantize_two_stage(ctypes.byref(w1), ctypes.byref(w2), 0x8000, None) == 2
    w1.in_ = (1 << 30) + 64
    assert lib.nf4_dequantize_two_stage(ctypes.byref(w1), ctypes.byref(w2), 0x8000, None) == 2
    # each side within 2^30 but their product past the 2^40-element limit: refused,
    # not quantized in part
    w1.out, w1.in_ = 1 << 30, (1 << 10) + 64
    assert lib.nf4_quantize_residual(0x1000, ctypes.byref(w1), q, 0x5000, 0x6000, None, None, 0x7000, 1 << 62,
                                     None) == 2
    w2.out, w2.in_ = w1.out, w1.in_
    assert lib.nf4_dequantize_two_stage(ctypes.byref(w1), ctypes.byref(w2), 0x8000, None) == 2


def test_codec_element_limit(lib):
    """Quantize and dequantize take at most 2^40 elements (out * in), checked without
    overflow however large each side is."""
    q = _lib.NF4QConfig(64, 0, 256)
    for out, inn in (((1 << 40) + 64, 1), (1 << 21, (1 << 19) + 64), ((1 << 62), 1 << 62)):
        assert lib.nf4_quantize(0x1000, _lib.DTYPE_BF16, out, inn, q, 0x2000, 0x3000, None, None, 0x4000, 256,
                                None) == 2
        w = _lib.QLoraWeight()
        w.out, w.in_, w.q = out, inn, q
        w.codes, w.absmax = 0x2000, 0x3000
        assert lib.nf4_dequantize(ctypes.byref(w), 0x5000, None) == 2


def test_linear_size_limits(lib):
    """M, in and out are limited to 2^20 (8192 counter tiles each: the backward's two
    concurrent split-K products use one half of the 16384 counters each)."""
    q = _lib.NF4QConfig(64, 0, 256)
    w = _lib.QLoraWeight()
    w.out, w.in_, w.q = 256, 256, q
    w.codes, w.absmax = 0x2000, 0x3000
    big = (1 << 20) + 128
    assert lib.qlora_linear_fwd(ctypes.byref(w), 0x1000, big, 0x1000, 0x1000, 16, 2.0, 0x1000, None, 0x4000,
                                1 << 40, None) == 2
    assert lib.qlora_linear_bwd(ctypes.byref(w), 0x1000, 0x1000, big, 0x1000, 0x1000, 16, 2.0, 0x1000, 0x1000,
                                0x1000, 0x1000, 0x4000, 1 << 40, None) == 2
    w.in_ = (1 << 20) + 256
    assert lib.qlora_linear_fwd(ctypes.byref(w), 0x1000, 8, 0x1000, 0x1000, 16, 2.0, 0x1000, None, 0x4000,
                                1 << 40, None) == 2


def test_workspace_sizes_reserve_the_counter_region(lib):
    """Entry points share one workspace per stream: bytes [256, 256 + 64 KiB) hold
    split-K counters that every call must find zero, so any call with scratch
    sizes its workspace past them (status 256 + counters 65536 + scratch)."""
    reserved = 256 + 65536
    n = 4096 * 4096
    assert lib.nf4_quantize_residual_workspace_size(n) >= reserved + 4 * n
    assert lib.qlora_lora_merge_requantize_workspace_size(4096, 4096) >= reserved + 4 * n // 64
    assert lib.qlora_fwd_workspace_size(8192, 4096, 4096, 16) >= reserved + 4096 * 64 * 4
    assert lib.qlora_bwd_workspace_size(8192, 4096, 4096, 16) >= reserved
    assert lib.qlora_lora_down_workspace_size(8192, 4096, 16) >= reserved + 8192 * 16 * 4
    nn = (ctypes.c_int64 * 2)(n, n)
    assert lib.nf4_layer_error_rank_workspace_size(2, nn) >= reserved + 2 * (n // 16384) * 16
    # the quantizer keeps only the status word and no scratch
    assert lib.nf4_quantize_workspace_size(n) == 256


def test_workspace_reset_argument_checks(lib):
    """qlora_reset_workspace (status word, split-K counters and the forward GEMM's
    block flags) refuses a missing or too-small workspace on the host; no device
    work is queued then."""
    assert lib.qlora_reset_workspace(None, 1 << 20, None) == 7     # QLORA_ERR_WORKSPACE
    buf = ctypes.create_string_buffer(64)
    assert lib.qlora_reset_workspace(ctypes.cast(buf, ctypes.c_void_p), 64, None) == 7
