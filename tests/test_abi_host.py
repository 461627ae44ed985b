"""The C-ABI library loads, exports every declared symbol, and validates
arguments on the host before touching a device (no GPU needed)."""
import ctypes
import os
import re

import pytest

import oracle
from compressive_fine_tuning_b200 import sk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sk.h")

SK_OK, SK_ERR_INVALID_ARG, SK_ERR_UNSUPPORTED, SK_ERR_CUDA = 0, 1, 2, 3

# fake, 16-byte aligned, non-overlapping "device" addresses: validation must
# reject bad calls before any of them is dereferenced
A = ctypes.c_void_p(0x10000000)
B = ctypes.c_void_p(0x20000000)
C = ctypes.c_void_p(0x30000000)
D = ctypes.c_void_p(0x40000000)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sk_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_expected_calls():
    names = declared_functions()
    for must in ("sk_pack", "sk_linear_fwd", "sk_linear_bwd_input", "sk_linear_bwd_lut"):
        assert must in names
    assert set(names) == set(sk.EXPORTED)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(sk._LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_strings():
    assert sk.lib.sk_abi_version() == 1
    for code, name in [(0, b"SK_OK"), (1, b"SK_ERR_INVALID_ARG"), (2, b"SK_ERR_UNSUPPORTED"),
                       (3, b"SK_ERR_CUDA"), (4, b"SK_ERR_DEVICE_CHECK"), (99, b"SK_ERR_UNKNOWN")]:
        assert sk.lib.sk_status_string(code) == name


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [32, 96, 160, 512, 1376, 4096, 5120, 11008, 13824, 28672])
def test_packed_sizes_match_oracle(bits, d):
    assert sk.packed_row_bytes(d, bits) == oracle.row_stride_bytes(d, bits)
    assert sk.packed_bytes(7, d, bits) == oracle.packed_bytes(7, d, bits)


def test_packed_sizes_reject_bad_args():
    assert sk.packed_row_bytes(33, 4) == 0
    assert sk.packed_row_bytes(64, 5) == 0
    assert sk.packed_bytes(-1, 64, 4) == 0


def fwd(packed=A, lut=B, bits=4, gpr=1, n=256, d=512, X=C, T=4, task=None, ntask=1, Y=D, ws=None, wsb=0):
    return sk.lib.sk_linear_fwd(packed, lut, bits, gpr, n, d, X, T, task, ntask, Y, ws, wsb, None)


def bwd_in(packed=A, lut=B, bits=4, gpr=1, n=256, d=512, dY=C, T=4, task=None, ntask=1, dX=D):
    return sk.lib.sk_linear_bwd_input(packed, lut, bits, gpr, n, d, dY, T, task, ntask, dX, None, 0, None)


def bwd_lut(packed=A, bits=4, gpr=1, n=256, d=512, X=B, dY=C, T=4, task=None, ntask=1, dlut=D, acc=0):
    return sk.lib.sk_linear_bwd_lut(packed, bits, gpr, n, d, X, dY, T, task, ntask, dlut, acc, None, 0, None)


@pytest.mark.parametrize("call", [fwd, bwd_in, bwd_lut])
@pytest.mark.parametrize("kw", [
    dict(bits=1), dict(bits=5), dict(n=0), dict(n=12), dict(d=48), dict(d=0), dict(gpr=0), dict(gpr=3),
    dict(gpr=32),  # 512 / 32 = 16 columns per group: not a multiple of 32
    dict(T=-1), dict(ntask=0),
])
def test_bad_shapes_rejected(call, kw):
    assert call(**kw) == SK_ERR_INVALID_ARG
    assert sk.lib.sk_last_error() != b""


def test_bad_pointers_rejected():
    assert fwd(packed=None) == SK_ERR_INVALID_ARG
    assert fwd(lut=None) == SK_ERR_INVALID_ARG
    assert fwd(X=None) == SK_ERR_INVALID_ARG
    assert fwd(Y=None) == SK_ERR_INVALID_ARG
    assert fwd(X=ctypes.c_void_p(0x30000008)) == SK_ERR_INVALID_ARG   # misaligned
    assert bwd_in(dX=ctypes.c_void_p(0x40000004)) == SK_ERR_INVALID_ARG
    assert bwd_lut(dlut=None) == SK_ERR_INVALID_ARG
    assert bwd_lut(dY=None) == SK_ERR_INVALID_ARG
    assert bwd_lut(acc=2) == SK_ERR_INVALID_ARG


def test_overlapping_output_rejected():
    # Y starts inside X's [T][d] bf16 range
    assert fwd(X=C, Y=ctypes.c_void_p(0x30000000 + 1024)) == SK_ERR_INVALID_ARG
    assert bwd_in(dY=C, dX=C) == SK_ERR_INVALID_ARG
    assert bwd_lut(X=B, dlut=ctypes.c_void_p(0x20000000 + 16)) == SK_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op():
    # T == 0 launches nothing, so it succeeds even without a device
    assert fwd(T=0) == SK_OK
    assert bwd_in(T=0) == SK_OK
    assert bwd_lut(T=0, acc=1) == SK_OK


def test_pack_validation():
    L = sk.lib
    assert L.sk_pack(A, 4, 64, 5, B, 4096, None) == SK_ERR_INVALID_ARG
    assert L.sk_pack(A, 4, 48, 4, B, 4096, None) == SK_ERR_INVALID_ARG
    assert L.sk_pack(A, 4, 64, 4, B, 16, None) == SK_ERR_INVALID_ARG           # buffer too small
    assert L.sk_pack(A, 0, 64, 4, B, 0, None) == SK_OK                          # nothing to do
    assert L.sk_pack(A, 4, 64, 4, ctypes.c_void_p(0x10000000 + 64), 4096, None) == SK_ERR_INVALID_ARG  # overlap
    assert L.sk_unpack(A, 4, 64, 7, B, None) == SK_ERR_INVALID_ARG
    assert L.sk_dequant(A, B, 4, 1, 256, 512, 1, 1, C, None) == SK_ERR_INVALID_ARG  # task outside [0, ntask)


def test_valid_call_without_device_fails_loudly():
    # the product path has no CPU fallback: with no usable device a valid call
    # reports a CUDA / unsupported-device error instead of computing anything
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    assert fwd() in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)
    assert bwd_in() in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)
    assert bwd_lut() in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)


def _adamw(**kw):
    a = dict(master=A, m=B, v=C, grad=ctypes.c_void_p(0x50000000), counts=None, ntask=1, n=8, gpr=2, bits=4,
             lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, step=1, lut=ctypes.c_void_p(0x60000000))
    a.update(kw)
    return sk.lib.sk_lut_adamw(a["master"], a["m"], a["v"], a["grad"], a["counts"], a["ntask"], a["n"], a["gpr"],
                               a["bits"], a["lr"], a["b1"], a["b2"], a["eps"], a["wd"], a["step"], a["lut"], None)


def test_lut_update_validation():
    assert _adamw(step=0) == SK_ERR_INVALID_ARG
    assert _adamw(b1=1.0) == SK_ERR_INVALID_ARG
    assert _adamw(b2=-0.1) == SK_ERR_INVALID_ARG
    assert _adamw(eps=0.0) == SK_ERR_INVALID_ARG
    assert _adamw(lr=float("nan")) == SK_ERR_INVALID_ARG
    assert _adamw(bits=5) == SK_ERR_INVALID_ARG
    assert _adamw(master=None) == SK_ERR_INVALID_ARG
    assert _adamw(v=ctypes.c_void_p(0x20000004)) == SK_ERR_INVALID_ARG           # misaligned
    assert _adamw(m=ctypes.c_void_p(0x10000000 + 64)) == SK_ERR_INVALID_ARG      # overlaps master
    assert _adamw(lut=ctypes.c_void_p(0x50000000 + 16)) == SK_ERR_INVALID_ARG    # overlaps grad
    L = sk.lib
    assert L.sk_lut_sgd(A, None, None, 1, 8, 2, 4, 0.1, None, None) == SK_ERR_INVALID_ARG
    assert L.sk_lut_sgd(A, B, None, 0, 8, 2, 4, 0.1, None, None) == SK_ERR_INVALID_ARG
    assert L.sk_bin_counts(A, 4, 3, 8, 64, B, None) == SK_ERR_INVALID_ARG        # gpr does not divide d
    assert L.sk_bin_counts(A, 4, 1, 8, 64, None, None) == SK_ERR_INVALID_ARG
    assert L.sk_bin_counts(A, 4, 1, 8, 64, ctypes.c_void_p(0x10000000 + 32), None) == SK_ERR_INVALID_ARG  # overlap


def test_lut_update_without_device_fails_loudly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    assert _adamw() in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)
    assert sk.lib.sk_lut_sgd(A, B, None, 1, 8, 2, 4, 0.1, None, None) in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)


E = ctypes.c_void_p(0x50000000)
F = ctypes.c_void_p(0x60000000)


def test_sketch_workspace_sizes():
    L = sk.lib
    assert L.sk_inverse_factor_workspace_bytes(4096) >= 4096 * 4096 * 8
    assert L.sk_inverse_factor_workspace_bytes(0) == 0
    assert L.sk_inverse_factor_workspace_bytes(1 << 17) == 0
    assert L.sk_sketch_round_workspace_bytes(4096, 4096) >= 4096 * 4096 * 8
    assert L.sk_sketch_round_workspace_bytes(0, 64) == 0


def test_sketch_validation():
    L = sk.lib
    big = 1 << 30
    # Gram: d >= 64 and a multiple of 8, pointers, aligned, no overlap
    assert L.sk_gram(A, 16, 60, B, 0, None) == SK_ERR_INVALID_ARG
    assert L.sk_gram(A, 16, 100, B, 0, None) == SK_ERR_INVALID_ARG
    assert L.sk_gram(A, -1, 64, B, 0, None) == SK_ERR_INVALID_ARG
    assert L.sk_gram(None, 16, 64, B, 0, None) == SK_ERR_INVALID_ARG
    assert L.sk_gram(A, 16, 64, ctypes.c_void_p(0x20000008), 0, None) == SK_ERR_INVALID_ARG
    assert L.sk_gram(A, 16, 64, ctypes.c_void_p(0x10000000 + 64), 0, None) == SK_ERR_INVALID_ARG
    # inverse factor: damp, workspace size, overlaps
    ws = L.sk_inverse_factor_workspace_bytes(64)
    assert L.sk_inverse_factor(A, 64, -0.1, B, C, D, ws, None) == SK_ERR_INVALID_ARG
    assert L.sk_inverse_factor(A, 64, float("inf"), B, C, D, ws, None) == SK_ERR_INVALID_ARG
    assert L.sk_inverse_factor(A, 64, 0.01, B, C, D, ws - 1, None) == SK_ERR_INVALID_ARG
    assert L.sk_inverse_factor(A, 64, 0.01, B, ctypes.c_void_p(0x20000000 + 64), D, ws, None) == SK_ERR_INVALID_ARG
    assert L.sk_inverse_factor(A, 0, 0.01, B, C, D, big, None) == SK_ERR_INVALID_ARG
    # Lloyd: bits, gpr dividing d, group length, max_iter
    assert L.sk_lloyd(A, B, 5, 1, 8, 64, 10, C, None, None) == SK_ERR_INVALID_ARG
    assert L.sk_lloyd(A, B, 4, 3, 8, 64, 10, C, None, None) == SK_ERR_INVALID_ARG
    assert L.sk_lloyd(A, B, 4, 1, 8, 32768, 10, C, None, None) == SK_ERR_UNSUPPORTED
    assert L.sk_lloyd(A, B, 4, 1, 8, 64, -1, C, None, None) == SK_ERR_INVALID_ARG
    assert L.sk_lloyd(A, B, 4, 1, 8, 64, 10, ctypes.c_void_p(0x10000000 + 16), None, None) == SK_ERR_INVALID_ARG
    # mapping: workspace size, overlaps
    wr = L.sk_sketch_round_workspace_bytes(8, 64)
    assert L.sk_sketch_round(A, B, C, 4, 1, 8, 64, D, E, wr - 1, None) == SK_ERR_INVALID_ARG
    assert L.sk_sketch_round(A, B, C, 4, 1, 8, 64, None, E, wr, None) == SK_ERR_INVALID_ARG
    assert L.sk_sketch_round(A, B, C, 4, 1, 8, 64, ctypes.c_void_p(0x30000000 + 16), E, wr, None) == SK_ERR_INVALID_ARG
    assert L.sk_sketch_round(A, B, C, 4, 2, 8, 63, D, E, wr, None) == SK_ERR_INVALID_ARG


def test_sketch_without_device_fails_loudly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    L = sk.lib
    assert L.sk_gram(A, 16, 64, B, 0, None) in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)
    assert L.sk_inverse_factor(A, 64, 0.01, B, C, D, L.sk_inverse_factor_workspace_bytes(64), None) in (
        SK_ERR_CUDA, SK_ERR_UNSUPPORTED)
    assert L.sk_lloyd(A, B, 4, 1, 8, 64, 10, C, None, None) in (SK_ERR_CUDA, SK_ERR_UNSUPPORTED)
    assert L.sk_sketch_round(A, B, C, 4, 1, 8, 64, D, E, L.sk_sketch_round_workspace_bytes(8, 64), None) in (
        SK_ERR_CUDA, SK_ERR_UNSUPPORTED)


C_PROGRAM = r"""
#include <stdio.h>
#include "sk.h"

/* a plain C caller: header compiles as C, symbols link without C++ mangling,
   and host-side validation answers before any device work */
int main(void) {
  if (sk_abi_version() != SK_ABI_VERSION) return 1;
  if (sk_packed_row_bytes(4096, 4) != 2048) return 2;
  if (sk_packed_bytes(7, 96, 3) != 7 * 48) return 3;
  if (sk_linear_fwd(NULL, NULL, 4, 1, 256, 512, NULL, 4, NULL, 1, NULL, NULL, 0, NULL) != SK_ERR_INVALID_ARG) return 4;
  if (sk_gram(NULL, 16, 60, NULL, 0, NULL) != SK_ERR_INVALID_ARG) return 5;
  if (sk_last_error()[0] == 0) return 6;
  printf("%s\n", sk_status_string(SK_ERR_INVALID_ARG));
  return 0;
}
"""


def test_c_caller_links_and_validates(tmp_path):
    """The header is valid C and the library links into a C program."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(sk._LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lsk", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip() == "SK_ERR_INVALID_ARG"


NOALLOC_REJECT = r"""
import ctypes, sys
sys.path.insert(0, sys.argv[1])
from compressive_fine_tuning_b200 import sk
# the 70B gate projection at 4 bits and 4 groups per row needs more partial-bin
# scratch than the allocation-free call holds, whatever the batch
n, d, bits, gpr, T = 28672, 8192, 4, 4, 64
need = sk.workspace_bytes(sk.SK_OP_BWD_LUT, n, d, bits, gpr, T, 1)
assert need > (32 << 20), need
p = [ctypes.c_void_p(a) for a in (0x10000000, 0x20000000, 0x40000000, 0x80000000)]
st = sk.lib.sk_linear_bwd_lut_noalloc(p[0], bits, gpr, n, d, p[1], p[2], T, None, 1, p[3], 0, None)
print(st, sk.lib.sk_last_error().decode())
"""


def test_noalloc_rejects_layers_beyond_its_scratch():
    """The allocation-free LUT gradient refuses, on the host, a layer whose
    partial bins exceed its fixed array.  The call runs in a child process that
    sees no CUDA device and keeps the library's own kernel choice, so even a
    broken size check could only fail on the missing device: nothing can be
    launched against the made-up addresses."""
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k != "SK_BWD_PATH"}
    env["CUDA_VISIBLE_DEVICES"] = ""
    r = subprocess.run([sys.executable, "-c", NOALLOC_REJECT, ROOT], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    st, msg = r.stdout.strip().split(" ", 1)
    assert int(st) == SK_ERR_INVALID_ARG
    assert "scratch" in msg


def test_group_validation():
    """The grouped forward checks every layer and the overlaps between layers
    on the host, before touching a device."""
    L = sk.lib
    mk = lambda p, lut, X, Y, n=256, d=512, gpr=1: sk._Layer(p, lut, gpr, n, d, X, Y)
    base = 0x10000000
    a = mk(base, base + 0x1000000, base + 0x2000000, base + 0x3000000)
    b = mk(base + 0x4000000, base + 0x5000000, base + 0x6000000, base + 0x7000000)
    arr = (sk._Layer * 9)(*([a, b] * 4 + [a]))
    assert L.sk_linear_fwd_group(arr, 0, 4, 4, None, 1, None) == SK_ERR_INVALID_ARG
    assert L.sk_linear_fwd_group(arr, 9, 4, 4, None, 1, None) == SK_ERR_INVALID_ARG
    assert L.sk_linear_fwd_group(None, 1, 4, 4, None, 1, None) == SK_ERR_INVALID_ARG
    bad = (sk._Layer * 2)(a, mk(base + 0x4000000, base + 0x5000000, base + 0x6000000, base + 0x3000000 + 16))
    assert L.sk_linear_fwd_group(bad, 2, 4, 4, None, 1, None) == SK_ERR_INVALID_ARG   # outputs overlap
    assert b"overlaps" in L.sk_last_error()
    reads = (sk._Layer * 2)(a, mk(base + 0x4000000, base + 0x5000000, base + 0x3000000, base + 0x7000000))
    assert L.sk_linear_fwd_group(reads, 2, 4, 4, None, 1, None) == SK_ERR_INVALID_ARG  # Y of one is X of another
    shape = (sk._Layer * 2)(a, mk(base + 0x4000000, base + 0x5000000, base + 0x6000000, base + 0x7000000, d=48))
    assert L.sk_linear_fwd_group(shape, 2, 4, 4, None, 1, None) == SK_ERR_INVALID_ARG
    assert b"layer 1" in L.sk_last_error()
    assert L.sk_linear_fwd_group(arr, 2, 4, 0, None, 1, None) == SK_OK                 # no tokens: nothing to do
