"""The C ABI from C (CPU only): include/specv.h compiles as C11 with warnings
as errors, a C program links against libspecv.so, and its host-side calls
(workspace sizes, status strings, argument rejection before any launch)
behave as the header states. No call here reaches the GPU."""
import os
import shutil
import subprocess

import pytest

import speculative_decoding_block_spec_b200 as specv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "specv.h"

static float host[64];  /* stands in for device buffers: never dereferenced, every call below is rejected first */

int main(void) {
  int bad = 0;
  void* p = host;
  if (spec_verify_workspace_size(8, 16, 1, 151936) == 0) bad = 1;
  if (spec_verify_workspace_size(0, 16, 1, 151936) != 0) bad = 2;           /* B < 1 */
  if (spec_verify_workspace_size(8, 16, SPEC_MAX_K + 1, 151936) != 0) bad = 3;
  if (spec_softmax_workspace_size(100) == 0) bad = 4;
  if (spec_dvl_workspace_size(32) == 0) bad = 5;
  if (strncmp(spec_status_string(SPEC_ERR_ARG), "SPEC_ERR_ARG", 12) != 0) bad = 6;
  /* null pointers */
  if (spec_verify_block(NULL, NULL, NULL, SPEC_BF16, NULL, NULL, NULL, NULL, 8, 16, 151936, 1.0f, NULL, NULL,
                        NULL, 0, NULL) != SPEC_ERR_ARG) bad = 7;
  /* T <= 0 */
  if (spec_verify_block(p, NULL, p, SPEC_F32, (int32_t*)p, NULL, host, host, 2, 2, 16, 0.0f, (int32_t*)p,
                        (int32_t*)p, p, 4096, NULL) != SPEC_ERR_ARG) bad = 8;
  /* K above SPEC_MAX_K */
  if (spec_verify_mixture(p, NULL, p, host, SPEC_MAX_K + 1, SPEC_F32, (int32_t*)p, NULL, host, host, 2, 2, 16,
                          1.0f, (int32_t*)p, (int32_t*)p, p, 4096, NULL) != SPEC_ERR_UNSUPPORTED) bad = 9;
  /* more rows than the fixed scratch of the allocation-free variant */
  if (spec_softmax_T_noalloc(p, SPEC_F32, SPEC_NOALLOC_MAX_ROWS + 1, 16, 16, 1.0f, host, host, NULL, NULL) !=
      SPEC_ERR_UNSUPPORTED) bad = 10;
  /* budget below the number of requests */
  if (dvl_allocate_pack(host, 4, 4, 3, (int32_t*)p, (int32_t*)p, NULL, NULL, NULL, SPEC_F32, 16, p, 4096, NULL) !=
      SPEC_ERR_ARG) bad = 11;
  if (bad) printf("bad %d\n", bad); else printf("ok\n");
  return bad;
}
"""


def test_header_compiles_as_c_and_host_calls_behave(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(specv.LIB_PATH)
    if not os.path.exists(specv.LIB_PATH):
        pytest.skip("libspecv.so is not built")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", lib_dir, "-lspecv", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    # no visible GPU: every call is rejected on the host, and one that were not could not launch
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
