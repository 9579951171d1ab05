"""The public header is a plain C interface: it compiles as C99 and as C++17
with warnings as errors, and a C caller can take the address of every entry
point with the declared signature.  Runs on the CPU (compile only)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
CUDA_INCLUDE = "/usr/local/cuda/include"

# A C translation unit that uses every declaration: taking each function's
# address into a pointer of the expected type makes a signature drift a
# compile error.
CALLER = r"""
#include "fa.h"
int use_all(void) {
  int (*f_fwd)(const void*, const void*, const void*, void*, float*, int, int, int, int, int, int,
               int, float, cudaStream_t) = fa_fwd;
  size_t (*f_ws)(int, int, int, int, int, int, int) = fa_bwd_workspace_size;
  const char* (*f_str)(int) = fa_status_string;
  int (*f_res)(const void*, const void*, const void*, void*, void*, float*, const fa_strides*,
               int, int, int, int, int, int, int, float, cudaStream_t) = fa_fwd_residual;
  int (*f_bres)(const void*, const void*, const void*, const void*, const void*, const float*,
                const void*, void*, void*, void*, const fa_strides*, int, int, int, int, int,
                int, int, float, void*, size_t, cudaStream_t) = fa_bwd_residual;
  fa_strides s = {1, 2, 3};
  (void)f_fwd; (void)f_ws; (void)f_str; (void)f_res; (void)f_bres; (void)s;
  return FA_OK + FA_MASK_BLOCK;
}
"""


def _compile(tmp_path, compiler, std, suffix):
    exe = shutil.which(compiler)
    if exe is None or not os.path.exists(os.path.join(CUDA_INCLUDE, "cuda_runtime_api.h")):
        pytest.skip(f"{compiler} or the CUDA headers are not available")
    src = tmp_path / f"caller{suffix}"
    src.write_text(CALLER)
    r = subprocess.run([exe, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                        "-I", INCLUDE, "-I", CUDA_INCLUDE, str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_header_constants_match_the_binding():
    """The binding's copies of the header's constants (mask block, the
    no-allocation scratch size) are the header's values."""
    import re
    from exact_io_aware_71_b200 import binding
    text = open(os.path.join(INCLUDE, "fa.h")).read()
    mb = int(re.search(r"#define FA_MASK_BLOCK (\d+)", text).group(1))
    m = re.search(r"#define FA_NOALLOC_SCRATCH_BYTES \((\d+)ull << (\d+)\)", text)
    assert mb == binding.MASK_BLOCK
    assert int(m.group(1)) << int(m.group(2)) == binding.NOALLOC_SCRATCH_BYTES


def test_header_compiles_as_c99(tmp_path):
    _compile(tmp_path, "gcc", "c99", ".c")


def test_header_compiles_as_cxx17(tmp_path):
    _compile(tmp_path, "g++", "c++17", ".cpp")
