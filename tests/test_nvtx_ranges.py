"""Every launching C-ABI entry point opens one NVTX range named after itself
and closes it on every return path (CPU only).

A small NVTX tool library (nvtx_recorder.c, built here with gcc) is loaded by
the NVTX loader through NVTX_INJECTION64_PATH in a child process and records
each push and pop.  The calls use argument sets that fail host-side validation
or are empty, so no call reaches CUDA; they exercise the early-return paths,
where a range left open would show as a missing pop.
"""
import json
import os
import shutil
import subprocess
import sys
from pathlib import Path

import pytest

import fp8_fine_grained_quant_b200 as fq

HERE = Path(__file__).resolve().parent
ROOT = HERE.parent

CHILD = r"""
import ctypes, json, sys
sys.path.insert(0, sys.argv[1])
import fp8_fine_grained_quant_b200 as fq
rec = ctypes.CDLL(sys.argv[2])
rec.rec_log.restype = ctypes.c_char_p
A16, A1 = 0x10000, 0x10001
calls = [
    ("fp8_quant_act_1x128", (A16, 4, 100, A16, A16, None)),
    ("fp8_quant_act_1x128_ue8m0", (A16, 0, 128, A16, A16, None)),
    ("fp8_quant_w_128x128", (None, 1, 128, 128, A16, A16, None)),
    ("fp8_quant_act_w", (A16, 4, 100, A16, A16, A16, 1, 128, 128, A16, A16, None)),
    ("fp8_quant_w_128x128_ue8m0", (A16, 1, 100, 128, A16, A16, None)),
    ("fp8_quant_act_128x1", (A16, 4, 128, A16, A1, None)),
    ("fp8_transpose_w_128x128", (A16, A16, 1, 128, 0, A16, A16, None)),
    ("fp8_gemm_blockscaled", (A16, A16, A16, A16, A16, 128, 256, 100, None)),
    ("fp8_gemm_unpromoted_diag", (A16, A16, A16, A16, A16, 0, 256, 128, None)),
    ("fp8_grouped_gemm_contiguous", (A16, A16, A16, A16, A1, A16, 256, 256, 128, 4, None)),
    ("fp8_grouped_gemm_masked", (A16, A16, A16, A16, A16, A16, 4, 200, 256, 128, 0, None)),
    ("fp8_swiglu_quant_1x128", (A16, 4, 100, None, 0, A16, A16, None)),
    ("fp8_quant_act_128x1_t", (A16, 4, 100, 128, A16, A16, None)),
    ("fp8_gemm_wgrad", (A16, A16, A16, A16, A16, 256, 256, 0, None)),
    ("fp8_mx_scales_act", (A16, 4, 100, A16, None)),
    ("fp8_mx_scales_w", (None, 1, 128, 128, A16, None)),
    ("fp8_gemm_mx", (A16, A16, A16, A16, A16, 0, 256, 128, None)),
    ("fp8_grouped_gemm_mx_contiguous", (A16, A16, A16, A16, A1, A16, 256, 256, 128, 4, None)),
    ("fp8_grouped_gemm_mx_masked", (A16, A16, A16, A16, A16, A16, 4, 200, 256, 128, None)),
]
out = []
lib = fq.lib()
for name, args in calls:
    rec.rec_clear()
    rc = getattr(lib, name)(*args)
    out.append({"name": name, "rc": rc, "log": rec.rec_log().decode(), "depth": rec.rec_depth()})
print(json.dumps(out))
"""


@pytest.fixture(scope="module")
def recorder(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out = tmp_path_factory.mktemp("nvtx") / "libnvtx_recorder.so"
    cuda_inc = Path(os.environ.get("CUDA_HOME", "/usr/local/cuda")) / "include"
    subprocess.run([cc, "-O1", "-shared", "-fPIC", "-I", str(cuda_inc), str(HERE / "nvtx_recorder.c"),
                    "-o", str(out)], check=True)
    return out


def test_every_entry_point_pushes_and_pops_one_named_range(recorder):
    fq.lib()  # the library is built
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(recorder), CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", CHILD, str(ROOT), str(recorder)], env=env,
                         capture_output=True, text=True, timeout=300, check=True)
    rows = json.loads(res.stdout.strip().splitlines()[-1])
    assert len(rows) == 19
    for r in rows:
        assert r["rc"] in (fq.OK, fq.ERR_SHAPE, fq.ERR_NULL, fq.ERR_ALIGN), r
        assert r["log"] == "push %s\npop\n" % r["name"], r
        assert r["depth"] == 0, r
    # the calls above span the status codes the early returns give
    assert {r["rc"] for r in rows} == {fq.OK, fq.ERR_SHAPE, fq.ERR_NULL, fq.ERR_ALIGN}
