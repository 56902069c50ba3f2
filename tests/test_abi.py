"""The C ABI library loads, exports every entry point include/kda.h declares, and
rejects bad arguments on the host (no GPU needed: these paths return before any
CUDA call)."""

import ctypes
import os
import re

import pytest

from gated_delta_rule_70_b200 import build, kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    hdr = open(os.path.join(ROOT, "include", "kda.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", hdr)))


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return kda.load_library()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("kda_prefill", "kda_decode_step", "kda_prefill_workspace_size", "kda_status_string",
              "kda_prologue", "kda_recurrence", "kda_prefill_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(kda.EXPORTED) >= set(_declared_functions())


def test_status_strings(lib):
    for code in range(6):
        s = kda.status_string(code)
        assert s.startswith("KDA_")
    assert "unknown" in kda.status_string(99)
    assert lib.kda_version() >= 100


def test_workspace_size_rules(lib):
    import torch
    record = 74752  # bytes per (chunk, head) record of the tensor-core path
    # bf16, d=128: chunk records only (the prologue runs inside chunk_prep)
    sh = kda.make_shape(4, 8192, 32, 128, torch.bfloat16)
    dense = kda.prefill_workspace_size(sh, False)
    varlen = kda.prefill_workspace_size(sh, True)
    T = 4 * 8192
    assert dense >= 4 * (8192 // 64) * 32 * record
    assert dense < 4 * (8192 // 64) * 32 * record + (1 << 20)
    assert varlen < dense  # 8192 packed tokens: ceil(8192/64) + 4 chunk slots
    # varlen: those slots' records, plus one 16-byte slot-table entry per slot and the
    # chunk table / sequence order
    slots = 8192 // 64 + 4
    assert varlen >= slots * 32 * record + slots * 16 + (4 + 1) * 4 + 4 * 4
    assert varlen < slots * 32 * record + (1 << 20)
    assert kda.recurrence_workspace_size(sh, False) == dense
    # a gate bound the chunk factorisation cannot hold takes the token kernel:
    # the prologue's intermediates, no records
    low = kda.make_shape(4, 8192, 32, 128, torch.bfloat16, lower_bound=-12.0)
    assert kda.prefill_workspace_size(low, False) >= T * 32 * 128 * (3 * 2 + 4) + T * 32 * 4
    assert kda.recurrence_workspace_size(low, False) < 4096
    # fp32 runs the standalone prologue, then a CUDA-core kernel: the prologue's intermediates
    f32 = kda.make_shape(1, 256, 2, 64, torch.float32)
    assert kda.prefill_workspace_size(f32, False) >= 256 * 2 * 64 * (3 * 4 + 4) + 256 * 2 * 4
    bad = kda.make_shape(4, 8192, 32, 96, torch.bfloat16)
    assert kda.prefill_workspace_size(bad, False) == 0


def _call_prefill(lib, shape, ptrs=None, ws=None, ws_bytes=0):
    P = ctypes.c_void_p
    x = P(256) if ptrs is None else ptrs
    return lib.kda_prefill(ctypes.byref(shape) if shape is not None else None,
                           x, x, x, x, x, x, x, x, None, None, None, x, x, None,
                           ws, ctypes.c_size_t(ws_bytes), None)


def test_host_validation_codes(lib):
    import torch
    ok = kda.make_shape(1, 16, 2, 64, torch.float32)
    assert _call_prefill(lib, None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert _call_prefill(lib, kda.make_shape(1, 16, 2, 96, torch.float32)) == kda.KDA_ERR_UNSUPPORTED
    assert _call_prefill(lib, kda.make_shape(1, 16, 65, 64, torch.float32)) == kda.KDA_ERR_UNSUPPORTED
    assert _call_prefill(lib, kda.make_shape(-1, 16, 2, 64, torch.float32)) == kda.KDA_ERR_INVALID_ARGUMENT
    bad_dtype = kda.make_shape(1, 16, 2, 64, torch.float32)
    bad_dtype.io_dtype = 7
    assert _call_prefill(lib, bad_dtype) == kda.KDA_ERR_INVALID_ARGUMENT
    bad_flags = kda.make_shape(1, 16, 2, 64, torch.float32)
    bad_flags.flags = 0x80
    assert _call_prefill(lib, bad_flags) == kda.KDA_ERR_INVALID_ARGUMENT
    nan_lb = kda.make_shape(1, 16, 2, 64, torch.float32, lower_bound=float("nan"))
    assert _call_prefill(lib, nan_lb) == kda.KDA_ERR_INVALID_ARGUMENT
    # a dense batch of more than 2^31 - 65 tokens: refused before any launch, no workspace size
    huge = kda.make_shape(65536, 65536, 2, 64, torch.float32)
    assert _call_prefill(lib, huge) == kda.KDA_ERR_UNSUPPORTED
    assert kda.prefill_workspace_size(huge, False) == 0
    assert kda.prefill_workspace_size(huge, True) > 0   # varlen: seq_len is the packed total
    # misaligned tensor pointer
    assert _call_prefill(lib, ok, ptrs=ctypes.c_void_p(258)) == kda.KDA_ERR_INVALID_ARGUMENT
    # missing / small / misaligned workspace
    assert _call_prefill(lib, ok) == kda.KDA_ERR_WORKSPACE
    assert _call_prefill(lib, ok, ws=ctypes.c_void_p(4096), ws_bytes=16) == kda.KDA_ERR_WORKSPACE
    assert _call_prefill(lib, ok, ws=ctypes.c_void_p(4096 + 16), ws_bytes=1 << 30) == kda.KDA_ERR_WORKSPACE
    # zero sequences: nothing to do
    assert _call_prefill(lib, kda.make_shape(0, 16, 2, 64, torch.float32)) == kda.KDA_OK


def test_decode_and_prologue_validation(lib):
    import torch
    P = ctypes.c_void_p
    x, nul = P(256), None
    sh = kda.make_shape(2, 1, 2, 128, torch.bfloat16)
    assert lib.kda_decode_step(ctypes.byref(sh), x, x, x, x, x, x, x, x, nul, x, x, None) \
        == kda.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_decode_step(ctypes.byref(kda.make_shape(2, 1, 2, 32, torch.bfloat16)),
                               x, x, x, x, x, x, x, x, x, x, x, None) == kda.KDA_ERR_UNSUPPORTED
    sh = kda.make_shape(1, 8, 2, 64, torch.float32)
    assert lib.kda_prologue(ctypes.byref(sh), x, x, x, x, x, x, x, x, None, None,
                            x, x, P(260), x, x, None, None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_recurrence(ctypes.byref(sh), x, x, x, x, x, None, None, x, None, x,
                              ctypes.c_size_t(1 << 20), None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_recurrence(ctypes.byref(sh), x, x, x, x, x, None, None, x, x, None,
                              ctypes.c_size_t(0), None) == kda.KDA_ERR_WORKSPACE


def test_binding_refuses_cpu_tensors(lib):
    import torch
    t = torch.zeros(16)
    with pytest.raises(ValueError):
        kda._ptr(t)


def test_output_gate_validation(lib):
    """kda_prefill_gated / kda_decode_step_gated reject a missing or misaligned gate or weight
    and a bad eps before any launch."""
    import torch
    P = ctypes.c_void_p
    x = P(256)
    sh = kda.make_shape(1, 16, 2, 64, torch.float32)
    def pre(og):
        return lib.kda_prefill_gated(ctypes.byref(sh), x, x, x, x, x, x, x, x, None, None, None,
                                     ctypes.byref(og), x, x, None, x, ctypes.c_size_t(1 << 30), None)
    assert pre(kda.OutputGate(None, 512, 1e-5)) == kda.KDA_ERR_INVALID_ARGUMENT
    assert pre(kda.OutputGate(264, 512, 1e-5)) == kda.KDA_ERR_INVALID_ARGUMENT
    assert pre(kda.OutputGate(512, 520, 1e-5)) == kda.KDA_ERR_INVALID_ARGUMENT
    assert pre(kda.OutputGate(512, 512, float("nan"))) == kda.KDA_ERR_INVALID_ARGUMENT
    assert pre(kda.OutputGate(512, 512, -1.0)) == kda.KDA_ERR_INVALID_ARGUMENT
    dsh = kda.make_shape(2, 1, 2, 128, torch.bfloat16)
    assert lib.kda_decode_step_gated(ctypes.byref(dsh), x, x, x, x, x, x, x, x,
                                     ctypes.byref(kda.OutputGate(None, 512, 1e-5)), x, x, x,
                                     None) == kda.KDA_ERR_INVALID_ARGUMENT


def test_decode_multi_validation(lib):
    import torch
    P = ctypes.c_void_p
    x = P(256)
    for T, want in ((0, kda.KDA_ERR_INVALID_ARGUMENT), (17, kda.KDA_ERR_INVALID_ARGUMENT)):
        sh = kda.make_shape(2, T, 2, 128, torch.bfloat16)
        assert lib.kda_decode_multi(ctypes.byref(sh), x, x, x, x, x, x, x, x, None, x, x, x, None,
                                    None) == want
    sh = kda.make_shape(2, 4, 2, 128, torch.bfloat16)
    assert lib.kda_decode_multi(ctypes.byref(sh), x, x, x, x, x, x, x, x, None, x, x, x, P(260),
                                None) == kda.KDA_ERR_INVALID_ARGUMENT


def test_missing_library_fails_loudly(monkeypatch):
    """Without libkda.so every call raises: there is no host fallback to run instead."""
    import torch
    monkeypatch.setattr(kda, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "libkda.so"))
    monkeypatch.setattr(kda, "_lib", None)
    with pytest.raises(kda.KdaLibraryError):
        kda.load_library()
    x = torch.zeros((64, 256), dtype=torch.bfloat16)
    with pytest.raises(kda.KdaLibraryError):
        kda.prefill(x, x, x, torch.zeros((3, 256, 4), dtype=torch.bfloat16),
                    torch.zeros((64, 2, 128), dtype=torch.bfloat16),
                    torch.zeros((64, 2), dtype=torch.bfloat16), torch.zeros(2), torch.zeros((2, 128)))
