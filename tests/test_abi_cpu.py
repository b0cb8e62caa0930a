"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, the binding refuses bad caller buffers, and every call rejects
invalid arguments on the host before touching a device.

The argument-validation cases pass fake, never-valid device addresses; a call
whose arguments are all valid must then stop at the device check.  They run in
a child process that sees no CUDA device (CUDA_VISIBLE_DEVICES set empty), so
on a machine with a GPU too no call can reach a kernel launch with those
addresses.  Nothing in this module launches device code."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import ternary_weight_linear_forward_b200 as bl
from ternary_weight_linear_forward_b200 import bitlinear as B



ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")

OK, NULL, SHAPE, ALIGN, DTYPE, WS, DEVICE, CUDA, TIMEOUT, ALIAS = range(10)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", src)))


def test_header_declares_the_four_core_calls():
    names = declared_functions()
    for core in ("bitlinear_quantize_weights", "bitlinear_pack", "bitlinear_quant_act", "bitlinear_forward"):
        assert core in names


def test_library_exports_every_declared_symbol():
    L = bl.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in B.SIGNATURES, f"binding lacks {name}"


def test_status_strings():
    for s in range(10):
        assert bl.status_string(s)
    assert bl.status_string(0) == "ok"
    assert bl.status_string(12345) == "unknown status"


def _L():
    return bl.lib()


def test_decode_engine_switch():
    L_ = _L()
    assert L_.bitlinear_get_decode_engine() == 0           # BL_ENGINE_AUTO initially
    assert L_.bitlinear_set_decode_engine(4) == SHAPE
    assert L_.bitlinear_set_decode_engine(-1) == SHAPE
    for name in ("cuda_cores", "tensor_cores", "cuda_cores_general", "auto"):
        with bl.decode_engine(name):
            assert bl.get_decode_engine() == name
    assert bl.get_decode_engine() == "auto"
    with pytest.raises(ValueError):
        bl.set_decode_engine("fpga")
    # the bounded-wait test hook is a host flag: set and withdrawn without a device
    assert L_.bitlinear_test_expire_next_wait(1) == OK
    assert L_.bitlinear_test_expire_next_wait(0) == OK


def test_binding_type_checks():
    import torch
    with pytest.raises(TypeError):
        bl.quant_act(torch.zeros(2, 64, dtype=torch.float16))
    with pytest.raises((TypeError, ValueError)):
        bl.pack(torch.zeros(2, 64, dtype=torch.int8))       # CPU tensor


def test_binding_checks_caller_buffers():
    # the binding knows tensor sizes, the C layer only pointers: a caller's
    # output, workspace, gamma or beta of the wrong size, dtype, device or
    # layout is refused before any library call
    import torch
    dev = torch.device("cpu")
    out = torch.empty((3, 5), dtype=torch.float32)
    B._check_out(out, (3, 5), B.FLOAT_OUT, dev)
    with pytest.raises(ValueError):
        B._check_out(out, (3, 6), B.FLOAT_OUT, dev)                 # too small for M x N
    with pytest.raises(ValueError):
        B._check_out(torch.empty((5, 3)), (3, 5), B.FLOAT_OUT, dev)  # transposed
    with pytest.raises(TypeError):
        B._check_out(out.to(torch.float16), (3, 5), B.FLOAT_OUT, dev)
    with pytest.raises(TypeError):
        B._check_out(out.numpy(), (3, 5), B.FLOAT_OUT, dev)
    with pytest.raises(ValueError):
        B._check_out(torch.empty((5, 3)).t(), (3, 5), B.FLOAT_OUT, dev)  # not contiguous
    with pytest.raises(ValueError):
        B._check_out(out, (3, 5), B.FLOAT_OUT, torch.device("cuda", 0))  # another device
    with pytest.raises(ValueError):
        B._check_len(torch.empty(2), (3,), "gamma")                   # short gamma
    with pytest.raises(ValueError):
        B._check_len(torch.empty(0), (1,), "beta")                    # empty beta
    with pytest.raises(ValueError):
        B._same_device(torch.device("cuda", 0), W_p=torch.empty(1))
    B._check_ws(None, dev)
    with pytest.raises(TypeError):
        B._check_ws(torch.empty(8, dtype=torch.int32), dev)
    with pytest.raises(ValueError):
        B._check_ws(torch.empty(8, dtype=torch.uint8), torch.device("cuda", 0))



def test_host_validation_in_a_process_without_a_device():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "abi_host_cases.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and " failed" not in r.stdout


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "bitlinear.h"

/* A plain C client: only calls whose arguments fail host validation, so
   nothing reaches a device. */
int main(void) {
    int bad = 0;
    if (strcmp(bitlinear_status_string(BL_OK), "ok") != 0) bad |= 1;
    if (bitlinear_forward(NULL, NULL, 1, 1024, NULL, NULL, 64, NULL, BL_F32, NULL, 0, NULL) != BL_ERR_NULL) bad |= 2;
    if (bitlinear_pack((const int8_t*)16, 4, 24, (uint32_t*)4096, NULL) != BL_ERR_SHAPE) bad |= 4;
    if (bitlinear_forward_workspace(2048, 4096, 4096) < 2048 * 4) bad |= 8;
    if (bitlinear_set_decode_engine(99) != BL_ERR_SHAPE) bad |= 16;
    if (bitlinear_forward_grouped_workspace(1, 64, 512, 3) != 0) bad |= 32;
    printf("%d\n", bad);
    return bad;
}
"""


def test_plain_c_client_compiles_links_and_runs():
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(B.LIB_PATH)
    out = os.path.join(libdir, "_build")          # the library's own (git-ignored) build folder
    os.makedirs(out, exist_ok=True)
    src = os.path.join(out, "abi_client.c")
    with open(src, "w") as f:
        f.write(C_CLIENT)
    exe = os.path.join(out, "abi_client")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                        "-L", libdir, "-l:libbitlinear.so", "-Wl,-rpath," + libdir, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "0", (r.returncode, r.stdout, r.stderr)
