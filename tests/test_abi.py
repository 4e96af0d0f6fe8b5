"""The C-ABI library: it loads without a GPU, exports every function that
include/qlora.h declares, and rejects bad arguments before launching anything
(these calls return before the library touches the CUDA runtime)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    with open(os.path.join(ROOT, "include", "qlora.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def q():
    from lora_fine_tuning_qlora_b200 import build
    build.build()
    from lora_fine_tuning_qlora_b200 import qlora
    return qlora


def test_header_declares_the_boundary():
    fns = _header_functions()
    for name in ("qlora_quantize_weight", "qlora_workspace_bytes", "qlora_forward",
                 "qlora_backward", "qlora_merge", "qlora_last_error"):
        assert name in fns


def test_library_exports_every_declared_symbol(q):
    lib = ctypes.CDLL(q.LIB_PATH)
    for name in _header_functions():
        assert hasattr(lib, name), name
    assert set(q.EXPORTED) == set(_header_functions())


def test_library_has_no_libcuda_or_torch_dependency(q):
    import subprocess
    out = subprocess.run(["ldd", q.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out
    assert "torch" not in out and "libc10" not in out


def test_version(q):
    assert "sm_100a" in q.version()


def test_workspace_bytes(q):
    d = q.desc(1024, 1024, 8, 8.0, __import__("torch").bfloat16)
    n = q.qlora_workspace_bytes(d, 1024)
    # at least the int8 copy of X and its scales
    assert n >= 1024 * 1024 + 4 * 1024
    assert n % 256 == 0
    bad = q.desc(1000, 1024, 8, 8.0, __import__("torch").bfloat16)  # K % 16 != 0
    assert q.qlora_workspace_bytes(bad, 1024) == 0


def _fwd(q, d, M, X=0x1000, Wq=0x2000, sw=0x3000, bias=None, A=0x4000, B=0x5000, Y=0x6000,
         xA=0x7000, ws=0x8000, wsb=1 << 30):
    P = ctypes.c_void_p
    return q.lib().qlora_forward(ctypes.byref(d) if d is not None else None, M, P(X), P(Wq), P(sw),
                                 P(bias) if bias else None, P(A), P(B), P(Y), P(xA), P(ws), wsb,
                                 None, None)


def test_forward_rejects_bad_arguments_without_launching(q):
    import torch
    d = q.desc(784, 128, 4, 4.0, torch.float32)
    assert _fwd(q, None, 64) == -1                       # NULL descriptor
    assert _fwd(q, d, -1) == -3                          # negative M
    assert _fwd(q, q.desc(784, 128, 0, 4.0, torch.float32), 64) == -3   # r = 0
    assert _fwd(q, q.desc(784, 128, 65, 4.0, torch.float32), 64) == -3  # r > 64
    assert _fwd(q, q.desc(780, 128, 4, 4.0, torch.float32), 64) == -5   # K % 16
    assert _fwd(q, q.desc(784, 0, 4, 4.0, torch.float32), 64) == -3     # N = 0
    assert _fwd(q, d, 64, X=0) == -1                     # NULL X
    assert _fwd(q, d, 64, X=0x1008) == -2                # X not 16-byte aligned
    assert _fwd(q, d, 64, ws=0x8010) == -2               # workspace not 256-byte aligned
    assert _fwd(q, d, 64, sw=0x3002) == -2               # fp32 vector misaligned
    assert b"aligned" in q.lib().qlora_last_error()
    assert _fwd(q, d, 64, wsb=16) == -1                  # workspace too small
    assert b"workspace" in q.lib().qlora_last_error()


def test_backward_and_merge_reject_bad_arguments(q):
    import torch
    P = ctypes.c_void_p
    d = q.desc(784, 128, 4, 4.0, torch.bfloat16)
    rc = q.lib().qlora_backward(ctypes.byref(d), 64, P(0x1000), None, P(0x2000), P(0x3000),
                                P(0x4000), P(0x5000), P(0x6000), None, P(0x7000), P(0x8000),
                                None, P(0x9000), 1 << 30, None)
    assert rc == -1  # NULL dY
    rc = q.lib().qlora_backward(ctypes.byref(d), 64, P(0x1000), P(0x1804), P(0x2000), P(0x3000),
                                P(0x4000), P(0x5000), P(0x6000), None, P(0x7000), P(0x8000),
                                None, P(0x9000), 1 << 30, None)
    assert rc == -2  # dY misaligned
    rc = q.lib().qlora_merge(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x4000),
                             P(0x1000), P(0x5000), None)
    assert rc == -1  # output aliases input
    rc = q.lib().qlora_merge(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x4000),
                             P(0x6008), P(0x5000), None)
    assert rc == -2  # Wq_out misaligned
    rc = q.lib().qlora_quantize_weight(P(0x1000), 784, 0, P(0x2000), P(0x3000), None)
    assert rc == -3


def test_binding_refuses_host_tensors(q):
    import torch
    W = torch.zeros((32, 16))
    with pytest.raises(ValueError):
        q.quantize_weight(W)


def test_rank_pass_rows_setting(q):
    """qlora_set_rank_pass_rows returns the previous setting and refuses
    negative values (no GPU needed)."""
    lib = q.lib()
    prev = lib.qlora_set_rank_pass_rows(256)
    assert prev == 0
    assert lib.qlora_set_rank_pass_rows(0) == 256
    assert lib.qlora_set_rank_pass_rows(-1) == -1
    assert b"rows per CTA" in lib.qlora_last_error()
    assert lib.qlora_set_rank_pass_rows(0) == 0


def test_int4_calls_reject_bad_arguments(q):
    """The packed int4 calls need K a multiple of 32 and 16-byte aligned code
    buffers; they refuse anything else before launching (fake pointers)."""
    import torch
    P = ctypes.c_void_p
    lib = q.lib()
    assert lib.qlora_quantize_weight_int4(P(0x1000), 48, 8, P(0x2000), P(0x3000), None) == -5
    assert lib.qlora_quantize_weight_int4(P(0x1000), 64, 8, P(0x2008), P(0x3000), None) == -2
    assert lib.qlora_quantize_weight_int4(None, 64, 8, P(0x2000), P(0x3000), None) == -1
    assert lib.qlora_unpack_int4(P(0x1000), 80, 8, P(0x2000), None) == -5
    assert lib.qlora_unpack_int4(P(0x1000), 64, 8, P(0x2004), None) == -2
    d = q.desc(784, 128, 4, 4.0, torch.bfloat16)  # K % 32 == 16
    assert lib.qlora_merge_int4(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x4000),
                                P(0x5000), P(0x6000), None) == -5
    assert lib.qlora_gemm_dx_int4(ctypes.byref(d), 64, P(0x1000), P(0x2000), P(0x3000), P(0x4000),
                                  P(0x5000), P(0x6000), 1 << 30, None) == -5
    assert b"multiple of 32" in lib.qlora_last_error()
    d = q.desc(1024, 128, 4, 4.0, torch.bfloat16)
    assert lib.qlora_merge_int4(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x4000),
                                P(0x1000), P(0x6000), None) == -1  # output aliases input


def test_int4_forward_rejects_k_not_multiple_of_32(q):
    import torch
    P = ctypes.c_void_p
    d = q.desc(784, 128, 4, 4.0, torch.bfloat16)
    rc = q.lib().qlora_gemm_forward_int4(ctypes.byref(d), 64, P(0x1000), P(0x2000), P(0x3000),
                                         P(0x4000), None, P(0x5000), P(0x6000), P(0x7000), None, None)
    assert rc == -5


def test_new_entry_points_reject_bad_arguments(q):
    """The outlier, float8 and permutation calls validate before any launch
    (fake device addresses are never dereferenced)."""
    lib = ctypes.CDLL(q.LIB_PATH)
    P = ctypes.c_void_p
    fake = P(4096)
    # permutation: not a permutation, too many axes, NULL
    sh = (ctypes.c_int64 * 2)(4, 4)
    assert lib.qlora_permute(fake, P(8192), 2, sh, (ctypes.c_int * 2)(0, 0), 4, None) == -1
    sh9 = (ctypes.c_int64 * 9)(*([2] * 9))
    assert lib.qlora_permute(fake, P(8192), 9, sh9, (ctypes.c_int * 9)(*range(9)), 4, None) == -3
    assert lib.qlora_permute(None, P(8192), 2, sh, (ctypes.c_int * 2)(1, 0), 4, None) == -1
    # float8 GEMM: K not a multiple of 16; unknown format
    lib.qlora_fp8_gemm.argtypes = [P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, P, P, P, P, ctypes.c_int, P]
    assert lib.qlora_fp8_gemm(fake, 0, fake, 0, 16, 16, 24, fake, fake, None, fake, 1, None) == -5
    assert lib.qlora_fp8_gemm(fake, 7, fake, 0, 16, 16, 32, fake, fake, None, fake, 1, None) == -1
    # the workspace variant: a misaligned workspace, and the same shape checks
    lib.qlora_fp8_gemm_ws.argtypes = [P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, P, P, P, P, ctypes.c_int, P, ctypes.c_size_t, P]
    assert lib.qlora_fp8_gemm_ws(fake, 0, fake, 0, 16, 16, 32, fake, fake, None, fake, 1, P(0x10010), 4096,
                                 None) == -2
    assert lib.qlora_fp8_gemm_ws(fake, 0, fake, 0, 16, 16, 24, fake, fake, None, fake, 1, None, 0, None) == -5
    # no split below one wave of pair tiles; a split where the last wave is partial
    assert q.qlora_fp8_gemm_workspace_bytes(256, 256, 1024) == 0
    assert q.qlora_fp8_gemm_workspace_bytes(0, 256, 1024) == 0
    # 4096 x 4096 outputs: 256 pair tiles on 74 pairs (148 SMs) leave 34 for a
    # partial last wave, split in halves: 34 tiles x 2 halves x 256 x 256 fp32
    assert q.qlora_fp8_gemm_workspace_bytes(4096, 4096, 16384) == 34 * 2 * 256 * 256 * 4
    # 16384 x 4096: 1024 tiles leave 62, too many to split in one wave of halves
    assert q.qlora_fp8_gemm_workspace_bytes(16384, 4096, 4096) == 0
    # a single 128-deep k-block cannot be split
    assert q.qlora_fp8_gemm_workspace_bytes(4096, 4096, 128) == 0
    # float8 quantizer: the next scale must not overwrite the one in use
    lib.qlora_fp8_quantize.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P,
                                       ctypes.c_int, P, P, P, ctypes.c_size_t, P]
    assert lib.qlora_fp8_quantize(fake, 4, 4, 1, 0, fake, fake, P(8192), 16, P(12288), None, P(16384), 256,
                                  None) == -1
    # float8 quantizer with column sums: layout it cannot take, short workspace
    lib.qlora_fp8_quantize_colsum.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P,
                                              P, ctypes.c_int, P, P, P, P, ctypes.c_size_t, P]
    need = q.qlora_fp8_colsum_workspace_bytes(300, 64)
    assert need == 256 + 4 * 3 * 64 and q.qlora_fp8_colsum_workspace_bytes(0, 64) == 0
    assert lib.qlora_fp8_quantize_colsum(fake, 300, 60, 1, 0, P(8192), P(8196), P(8448), 16, P(12288), None,
                                         P(16384), P(32768), need, None) == -5   # cols % 8 != 0
    assert lib.qlora_fp8_quantize_colsum(fake, 300, 64, 1, 0, P(8192), P(8196), P(8448), 16, P(12288),
                                         P(65536), P(16384), P(32768), need, None) == -5  # rows % 16 != 0 with qt
    assert lib.qlora_fp8_quantize_colsum(fake, 300, 64, 1, 0, P(8192), P(8196), P(8448), 16, P(12288), None,
                                         P(16384), P(32768), need - 1, None) == -1
    assert lib.qlora_fp8_quantize_colsum(fake, 300, 64, 1, 0, P(8192), P(8196), P(8448), 16, P(12288), None,
                                         P(16384), P(32772), need, None) == -2   # workspace not 256-aligned
    # outlier kernel: capacity below the bound, NULL member
    cap = q.qlora_outlier_cap(256, 256)
    assert cap == (int((256 * 256 - 1) * 0.1 / 100) + 1) + (256 * 256 - 1 - int((256 * 256 - 1) * 99.9 / 100))
    ok = q.OutlierKernelStruct(4096, 8192, 12288, 16384, 20480, 24576, 28672, cap)
    small = q.OutlierKernelStruct(4096, 8192, 12288, 16384, 20480, 24576, 28672, cap - 1)
    ws = P(32768)
    nbytes = q.qlora_outlier_workspace_bytes(256, 256)
    assert lib.qlora_outlier_quantize(fake, 256, 256, ctypes.byref(small), ws, nbytes, None) == -1
    nul = q.OutlierKernelStruct(4096, 0, 12288, 16384, 20480, 24576, 28672, cap)
    assert lib.qlora_outlier_quantize(fake, 256, 256, ctypes.byref(nul), ws, nbytes, None) == -1
    assert lib.qlora_outlier_quantize(fake, 256, 256, ctypes.byref(ok), ws, nbytes - 1, None) == -1
    # the outlier layer refuses a K that is not a multiple of 16
    d = q.desc(100, 64, 4, 4.0, __import__("torch").bfloat16)
    assert lib.qlora_outlier_forward(ctypes.byref(d), 8, fake, ctypes.byref(ok), None, fake, fake, fake, fake,
                                     ws, 1 << 20, None) == -5
