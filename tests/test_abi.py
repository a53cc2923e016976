"""The C-ABI library: it loads, exports every function include/nvfp4.h declares, and its host-side
logic (scale layout helpers, tile choice, argument checks) behaves as documented.  No GPU needed:
every call here returns before the first CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

from epilogue_gemm_nvfp4_b200 import binding as B
from oracle import nvfp4_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(B.EXPORTS)


def test_library_loads_and_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.nvfp4_version() >= 100
    assert B.status_string(B.ERR_MISALIGNED).startswith("misaligned")


def test_scale_helpers_match_the_layout_definition(lib):
    for rows, cols in [(1, 16), (127, 64), (128, 512), (300, 208), (4608, 4608)]:
        assert lib.nvfp4_scale_bytes(rows, cols) == O.scale_buffer_bytes(rows, cols)
    rng = np.random.default_rng(0)
    for _ in range(200):
        rows, cols = int(rng.integers(1, 2000)), int(rng.integers(1, 400)) * 16
        r, kb = int(rng.integers(0, rows)), int(rng.integers(0, cols // 16))
        assert lib.nvfp4_scale_offset(r, kb, cols) == O.scale_atom_offset(r, kb, cols)


def test_scale_atoms_form_the_rows_the_gemm_tma_reads(lib):
    """The pair GEMM loads block scales with TMA over the scale bytes viewed as rows of one 512-byte
    atom: row b * k_atoms + k holds the scales of blocks 4k..4k+3 of rows 128b..128b+127, so the scales
    of one stage (four K atoms of one 128-row block) are a box of four consecutive rows, and a tensor's
    scale buffer is a whole number of such rows."""
    rng = np.random.default_rng(1)
    for cols in (64, 272, 4608, 12288, 53248):
        k_atoms = (cols // 16 + 3) // 4
        for _ in range(300):
            r, kb = int(rng.integers(0, 1000)), int(rng.integers(0, cols // 16))
            assert lib.nvfp4_scale_offset(r, kb, cols) // 512 == (r // 128) * k_atoms + kb // 4
        for rows in (1, 128, 1000):
            assert lib.nvfp4_scale_bytes(rows, cols) == (rows + 127) // 128 * k_atoms * 512


def test_tile_choice_depends_on_n_k_kind_only(lib):
    assert B.tile_n(13824, 4608, "qknorm") == 256
    assert B.tile_n(24576, 4608, "gated_silu") == 256
    assert B.tile_n(4608, 53248, "bias") in (128, 256)
    assert B.tile_n(384, 512, "bias") == 128
    assert B.tile_n(384, 512, "qknorm") == 0          # heads need 256-column tiles
    assert B.tile_n(512, 96, "bias") == 0             # K % 64
    assert B.tile_n(200, 512, "bias") == 0            # N % 16
    assert B.tile_n(400, 512, "bias") == 128          # ragged last tile
    assert B.tile_n(4624, 4608, "resid_gate") == 128
    assert B.tile_n(400, 512, "gated_silu") == 0      # a and b halves pair 128-row blocks


def _tensor(rows, cols, ptr=0x10000):
    return B.CTensor(ptr, ptr, ptr, rows, cols, cols // 2)


def test_argument_checks_return_before_any_launch(lib):
    desc = B.CEpilogue()
    a, w = _tensor(256, 512), _tensor(512, 512)
    lin = lambda a_, w_, d_, out=0x10000, ld=512, q=None: lib.nvfp4_linear(
        ctypes.byref(a_), ctypes.byref(w_), ctypes.byref(d_), out, ld, q, None)
    assert lib.nvfp4_linear(None, ctypes.byref(w), ctypes.byref(desc), 0x10000, 512, None, None) == B.ERR_INVALID_ARG
    assert lin(_tensor(256, 512), _tensor(512, 256), desc) == B.ERR_INVALID_ARG          # K mismatch
    assert lin(_tensor(256, 96), _tensor(512, 96), desc) == B.ERR_UNSUPPORTED_SHAPE      # K % 64
    assert lin(_tensor(256, 512), _tensor(200, 512), desc) == B.ERR_UNSUPPORTED_SHAPE    # N % 16
    assert lin(_tensor(256, 512, 0x10008), w, desc) == B.ERR_MISALIGNED
    assert lin(a, w, desc, out=0x10002) == B.ERR_MISALIGNED
    assert lin(a, w, desc, ld=100) == B.ERR_INVALID_ARG                                    # ld_out < N
    assert lin(a, w, desc, out=0) == B.ERR_INVALID_ARG                                     # no output at all
    bad = B.CEpilogue(kind=7)
    assert lin(a, w, bad) == B.ERR_INVALID_ARG
    qk = B.CEpilogue(kind=B.EPI_QKNORM, gamma_q=0x10000, gamma_k=0x10000, eps=1e-6, head_dim=128)
    assert lin(a, w, qk) == B.ERR_INVALID_ARG                                              # head_dim != 256
    qk = B.CEpilogue(kind=B.EPI_QKNORM, gamma_q=0x10000, gamma_k=0x10000, eps=1e-6, head_dim=256,
                     q_col0=0, k_col0=256, qk_cols=512)
    assert lin(a, w, qk) == B.ERR_UNSUPPORTED_SHAPE                                        # k range past N
    rg = B.CEpilogue(kind=B.EPI_RESID_GATE)
    assert lin(a, w, rg) == B.ERR_INVALID_ARG                                              # no residual/gate
    q = _tensor(256, 256)
    gs = B.CEpilogue(kind=B.EPI_GATED_SILU, out_nvfp4=1)
    assert lin(a, w, gs, q=ctypes.byref(_tensor(256, 512))) == B.ERR_INVALID_ARG           # out_fp4 not [M, N/2]
    # empty and oversized problems: M = 0 is a valid call that launches nothing (so it succeeds even
    # without a device); a dimension past 2^30 is refused
    assert lin(_tensor(0, 512), w, desc, out=0x10000) == B.OK
    big = 1 << 30
    assert lin(_tensor(big + 1, 512), w, desc) == B.ERR_UNSUPPORTED_SHAPE                 # M > 2^30
    assert lin(_tensor(256, 512), _tensor(big + 256, 512), desc, ld=big + 256) == B.ERR_UNSUPPORTED_SHAPE
    assert lin(_tensor(256, big + 64), _tensor(512, big + 64), desc) == B.ERR_UNSUPPORTED_SHAPE
    # quantise / dequantise / amax
    t = _tensor(4, 512)
    assert lib.nvfp4_quantize(None, 4, 512, 512, 1, ctypes.byref(t), None) == B.ERR_INVALID_ARG
    assert lib.nvfp4_quantize(0x10000, 4, 520, 520, 1, ctypes.byref(_tensor(4, 520)), None) == B.ERR_UNSUPPORTED_SHAPE
    assert lib.nvfp4_quantize(0x10000, 4, 512, 500, 1, ctypes.byref(t), None) == B.ERR_INVALID_ARG
    assert lib.nvfp4_quantize(0x10000, 4, 512, 516, 1, ctypes.byref(t), None) == B.ERR_MISALIGNED
    assert lib.nvfp4_quantize(0x10000, 5, 512, 512, 1, ctypes.byref(t), None) == B.ERR_INVALID_ARG
    assert lib.nvfp4_dequantize(ctypes.byref(t), None, 512, None) == B.ERR_INVALID_ARG
    assert lib.nvfp4_amax(0x10000, 4, 512, 512, None, None) == B.ERR_INVALID_ARG
    # fused output amax: a 4-byte aligned fp32 slot
    am = B.CEpilogue(out_amax=0x10002)
    assert lin(a, w, am) == B.ERR_MISALIGNED
    # fake quantisation
    fq = lambda x=0x10000, rows=4, cols=512, ldx=512, cs=1, g=0x10000, y=0x10000, ldy=512: \
        lib.nvfp4_fake_quantize(x, rows, cols, ldx, cs, g, y, ldy, None)
    assert fq(x=None) == B.ERR_INVALID_ARG
    assert fq(y=None) == B.ERR_INVALID_ARG
    assert fq(g=None) == B.ERR_INVALID_ARG
    assert fq(cols=520, ldx=520, ldy=520) == B.ERR_UNSUPPORTED_SHAPE                     # cols % 16
    assert fq(ldy=256) == B.ERR_INVALID_ARG                                                 # ldy < cols
    assert fq(y=0x10008) == B.ERR_MISALIGNED
    assert fq(ldx=516) == B.ERR_MISALIGNED
    assert fq(g=0x10001) == B.ERR_MISALIGNED
    # adaLN prologue of the quantiser
    ok = dict(shift=0x10000, scale=0x10000, ld_mod=512, rows_per_sample=0, eps=1e-6, rstd=0x10000,
              u_out=0x10000, ld_u=512)

    def ada(x=0x10000, rows=4, cols=512, ldx=512, t=t, **kw):
        d = B.CAdaln(**dict(ok, **kw))
        return lib.nvfp4_adaln_quantize(x, rows, cols, ldx, ctypes.byref(d), 1, ctypes.byref(t), None)
    assert lib.nvfp4_adaln_quantize(0x10000, 4, 512, 512, None, 1, ctypes.byref(t), None) == B.ERR_INVALID_ARG
    assert ada(x=None) == B.ERR_INVALID_ARG
    assert ada(eps=0.0) == B.ERR_INVALID_ARG
    assert ada(eps=float("nan")) == B.ERR_INVALID_ARG
    assert ada(rows_per_sample=-1) == B.ERR_INVALID_ARG
    assert ada(rows_per_sample=2, ld_mod=256) == B.ERR_INVALID_ARG                        # samples overlap
    assert ada(ld_u=256) == B.ERR_INVALID_ARG
    assert ada(rows=5) == B.ERR_INVALID_ARG                                                # out is [4, 512]
    assert ada(cols=520, ldx=520, ld_u=520, t=_tensor(4, 520)) == B.ERR_UNSUPPORTED_SHAPE
    assert ada(ldx=516) == B.ERR_MISALIGNED
    assert ada(shift=0x10008) == B.ERR_MISALIGNED
    assert ada(scale=0x10004) == B.ERR_MISALIGNED
    assert ada(rows_per_sample=2, ld_mod=516) == B.ERR_MISALIGNED
    assert ada(rstd=0x10002) == B.ERR_MISALIGNED
    assert ada(u_out=0x10008) == B.ERR_MISALIGNED
    assert ada(ld_u=516) == B.ERR_MISALIGNED
    # W8A8 INT8
    i8 = lambda rows, cols, ptr=0x10000, ld=0, scale=0x10000: B.CInt8Tensor(ptr, scale, rows, cols, ld)
    iq = lambda x=0x10000, rows=4, cols=512, ldx=512, mult=None, t=None: lib.nvfp4_int8_quantize(
        x, rows, cols, ldx, mult, ctypes.byref(t if t is not None else i8(rows, cols)), None)
    assert iq(x=None) == B.ERR_INVALID_ARG
    assert iq(t=i8(5, 512)) == B.ERR_INVALID_ARG                                         # rows differ
    assert iq(cols=520, ldx=520, t=i8(4, 520, ld=528)) == B.ERR_UNSUPPORTED_SHAPE
    assert iq(ldx=516) == B.ERR_MISALIGNED
    assert iq(mult=0x10004) == B.ERR_MISALIGNED
    assert iq(t=i8(4, 512, ld=520)) == B.ERR_MISALIGNED                                   # ld % 16
    assert iq(t=i8(4, 512, scale=0x10002)) == B.ERR_MISALIGNED
    assert lib.nvfp4_int8_quantize(0x10000, 4, 512, 512, None, None, None) == B.ERR_INVALID_ARG
    il = lambda a_, w_, d_=desc, out=0x10000, ld=512: lib.nvfp4_int8_linear(
        ctypes.byref(a_), ctypes.byref(w_), ctypes.byref(d_), out, ld, None, None)
    assert il(i8(256, 512), i8(512, 256)) == B.ERR_INVALID_ARG                            # K mismatch
    assert il(i8(256, 48), i8(512, 48)) == B.ERR_UNSUPPORTED_SHAPE                        # K % 32
    assert il(i8(256, 512), i8(200, 512)) == B.ERR_UNSUPPORTED_SHAPE                      # N % 128
    assert il(i8(256, 512, scale=0x10004), i8(512, 512)) == B.ERR_MISALIGNED              # scales 16-byte aligned
    assert il(i8(256, 512), i8(512, 512), out=0x10002) == B.ERR_MISALIGNED
    assert il(i8(256, 512), i8(512, 512), d_=B.CEpilogue(kind=9)) == B.ERR_INVALID_ARG


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_cuda_error(lib):
    a, w = _tensor(256, 512), _tensor(512, 512)
    desc = B.CEpilogue()
    assert lib.nvfp4_linear(ctypes.byref(a), ctypes.byref(w), ctypes.byref(desc), 0x10000, 512, None, None) \
        == B.ERR_CUDA
    a8, w8 = B.CInt8Tensor(0x10000, 0x10000, 256, 512, 0), B.CInt8Tensor(0x10000, 0x10000, 512, 512, 0)
    assert lib.nvfp4_int8_linear(ctypes.byref(a8), ctypes.byref(w8), ctypes.byref(desc), 0x10000, 512, None, None) \
        == B.ERR_CUDA


def test_ctypes_structs_match_the_header(tmp_path):
    """The binding's ctypes structs have the C header's field offsets and sizes (compiled with gcc)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    structs = {"nvfp4_tensor": B.CTensor, "nvfp4_epilogue_desc": B.CEpilogue, "nvfp4_adaln_desc": B.CAdaln,
               "nvfp4_int8_tensor": B.CInt8Tensor}
    lines = ['#include <stdio.h>', '#include "nvfp4.h"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines.append("  return 0;\n}")
    src = tmp_path / "layout.c"
    exe = tmp_path / "layout"
    src.write_text("\n".join(lines))
    subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        cname, what, value = line.split()
        got[(cname, what)] = int(value)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert got[(cname, field)] == getattr(py, field).offset, (cname, field)


def test_c_program_links_and_calls_the_abi(tmp_path):
    """A plain C program, compiled with gcc against include/nvfp4.h and linked with libnvfp4.so, calls the
    host helpers and gets the documented argument errors (no device needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib_dir = os.path.dirname(B.LIB_PATH)
    src = tmp_path / "use.c"
    src.write_text(r'''
#include <stdio.h>
#include "nvfp4.h"
int main(void) {
  nvfp4_tensor t = {(void*)0x10000, (void*)0x10000, (float*)0x10000, 4, 520, 0};
  nvfp4_epilogue_desc epi = {0};
  nvfp4_tensor a = {(void*)0x10000, (void*)0x10000, (float*)0x10000, 256, 512, 0};
  nvfp4_tensor w = {(void*)0x10000, (void*)0x10000, (float*)0x10000, 200, 512, 0};
  printf("%zu %lld %d %d %d %s\n", nvfp4_scale_bytes(300, 208), (long long)nvfp4_scale_offset(130, 5, 208),
         (int)nvfp4_quantize((void*)0x10000, 4, 520, 520, 1, &t, NULL),
         (int)nvfp4_linear(&a, &w, &epi, (void*)0x10000, 512, NULL, NULL),
         (int)nvfp4_linear_tile_n(13824, 4608, NVFP4_EPI_QKNORM), nvfp4_status_string(NVFP4_ERR_MISALIGNED));
  return 0;
}
''')
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe), "-L", lib_dir,
                    "-lnvfp4", f"-Wl,-rpath,{lib_dir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert int(out[0]) == O.scale_buffer_bytes(300, 208)
    assert int(out[1]) == O.scale_atom_offset(130, 5, 208)
    assert int(out[2]) == B.ERR_UNSUPPORTED_SHAPE          # cols % 16
    assert int(out[3]) == B.ERR_UNSUPPORTED_SHAPE          # N % 16
    assert int(out[4]) == 256
    assert " ".join(out[5:]).startswith("misaligned")
