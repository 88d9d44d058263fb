"""The C-ABI library loads without a GPU, exports every symbol the header
declares, sizes workspaces, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_27_b200 import gq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    txt = open(os.path.join(ROOT, "include", "gq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(gq_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = gq.lib()
    names = _header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(gq.EXPORTS) <= set(names)


def test_status_strings_and_counter():
    L = gq.lib()
    assert L.gq_status_string(0) == b"GQ_OK"
    assert L.gq_status_string(5) == b"GQ_ERR_NOT_PD"
    assert gq.launch_count() >= 0


def test_workspace_sizes():
    assert gq.hessian_workspace_size(2048, 768) > 256
    assert gq.hessian_workspace_size(0, 768) >= 256
    assert gq.hessian_workspace_size(10, 7) == 0
    assert gq.damp_cholesky_workspace_size(768) > 0
    assert gq.gptq_workspace_size(768, 768, 128) > 0
    assert gq.recon_workspace_size(768, 768, 2048) > 0


FAKE = ctypes.c_void_p(4096)   # never dereferenced: every call below fails validation


@pytest.mark.parametrize("args,code", [
    # bad dtype
    (dict(dt=7, d_out=8, d_in=8, bits=4, g=-1, sym=1), 3),
    # d_in not a multiple of 8
    (dict(dt=0, d_out=8, d_in=12, bits=4, g=-1, sym=1), 2),
    # group does not divide d_in
    (dict(dt=0, d_out=8, d_in=64, bits=4, g=48, sym=1), 2),
    # an unsupported code width
    (dict(dt=0, d_out=8, d_in=64, bits=5, g=-1, sym=1), 1),
    # 3-bit codes need d_in a multiple of 32
    (dict(dt=0, d_out=8, d_in=72, bits=3, g=-1, sym=1), 2),
    # 8-bit codes need the group a multiple of 32
    (dict(dt=0, d_out=8, d_in=64, bits=8, g=16, sym=1), 2),
    # affine without zeros
    (dict(dt=0, d_out=8, d_in=64, bits=4, g=-1, sym=0), 1),
])
def test_rtn_argument_errors(args, code):
    L = gq.lib()
    st = L.gq_rtn_quantize_pack(FAKE, args["dt"], args["d_out"], args["d_in"], args["bits"],
                                args["g"], args["sym"], FAKE, FAKE, None, None)
    assert st == code
    assert L.gq_last_error() != b""


def test_other_argument_errors():
    L = gq.lib()
    # null H
    assert L.gq_hessian_accumulate(FAKE, 64, 64, None, FAKE, 1 << 20, None) == 1
    # workspace too small
    assert L.gq_hessian_accumulate(FAKE, 64, 64, FAKE, FAKE, 8, None) == 4
    # act_order without perm_out
    assert L.gq_damp_cholesky_inverse(FAKE, 64, 0.01, 1, None, None, FAKE, None, None,
                                      FAKE, 1 << 30, None) == 1
    # negative damping
    assert L.gq_damp_cholesky_inverse(FAKE, 64, -1.0, 0, None, None, FAKE, None, None,
                                      FAKE, 1 << 30, None) == 1
    # H or U not 16-byte aligned (the row kernels read them as float4)
    odd = ctypes.c_void_p(4096 + 4)
    assert L.gq_damp_cholesky_inverse(odd, 64, 0.01, 0, None, None, FAKE, None, None,
                                      FAKE, 1 << 30, None) == 1
    assert L.gq_damp_cholesky_inverse(FAKE, 64, 0.01, 0, None, None, odd, None, None,
                                      FAKE, 1 << 30, None) == 1
    assert L.gq_damp_cholesky_inverse_noalloc(odd, 64, 0.01, 0, None, None, FAKE, None,
                                              None, None) == 1
    # group_size must divide block_size
    assert L.gq_gptq_quantize_layer(FAKE, 0, 8, 192, FAKE, 4, 48, 96, 1, None, None,
                                    FAKE, FAKE, None, None, FAKE, 1 << 40, None) == 1
    # misaligned workspace
    assert L.gq_gptq_quantize_layer(FAKE, 0, 8, 128, FAKE, 4, 128, 128, 1, None, None, FAKE,
                                    FAKE, None, None, ctypes.c_void_p(4096 + 8), 1 << 40,
                                    None) == 4
    # recon: null sse_dev
    assert L.gq_recon_error(FAKE, 0, FAKE, FAKE, None, None, 8, 64, 4, -1, 1, FAKE, 16, None,
                            None, None, FAKE, 1 << 30, None) == 1
    # GPTQ at another width than 4 bits needs block 128
    assert L.gq_gptq_quantize_layer(FAKE, 0, 8, 128, FAKE, 8, 64, 64, 1, None, None,
                                    FAKE, FAKE, None, None, FAKE, 1 << 40, None) == 1
    # trace route: null H0
    assert L.gq_recon_error_hessian(FAKE, 0, FAKE, FAKE, None, None, 8, 64, 4, -1, 1, None, 16,
                                    FAKE, None, None, FAKE, 1 << 30, None) == 1


def test_kernel_timer_without_session():
    L = gq.lib()
    assert L.gq_kernel_timer_start(1, 0) == 1       # capacity must be positive
    assert L.gq_kernel_timer_start(1, -5) == 1
    assert L.gq_kernel_timer_read(None, None, None, 0) == 0
    assert L.gq_kernel_timer_stop() == 0
    assert L.gq_kernel_timer_release() == 0
    assert set(gq.KERNEL_UNITS) == set(gq.KERNELS)


def test_header_is_c_and_links_from_c(tmp_path):
    """include/gq.h compiles as C99 and a C program links libgq.so and calls
    it (the calls below need no GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_gq.c"
    src.write_text(
        '#include "gq.h"\n#include <stdio.h>\n'
        "int main(void) {\n"
        '  printf("%s %zu %zu\\n", gq_status_string(GQ_ERR_NOT_PD),\n'
        "         gq_hessian_workspace_size(2048, 768), gq_awq_workspace_size(8, 64, 16, 4, -1, 1));\n"
        "  return gq_rtn_quantize_pack(0, GQ_F32, 8, 64, 4, -1, 1, 0, 0, 0, 0) == GQ_ERR_ARG ? 0 : 1;\n"
        "}\n")
    libdir = os.path.dirname(gq.LIB_PATH)
    exe = tmp_path / "use_gq"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lgq", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[0] == "GQ_ERR_NOT_PD" and int(out[1]) > 0 and int(out[2]) > 0
