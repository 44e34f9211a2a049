"""The kernel variants the library selects from its environment, each run through the
whole-stack parity tests in a child process (the switches are read once per process):

  WK_FUSED_LN=1     residual + output LayerNorm inside the last FMB Linear and LCB epilogues
  WK_FM_MMA_SYNC=1  the FM + LayerNorm on warp-level mma.sync instead of tcgen05
  WK_PAIR_GEMM=0    the FMB MLP on one-CTA tcgen05 tiles instead of CTA pairs
  WK_RES_LN_RING=0  the residual + LayerNorm without the bulk-copy ring
  WK_LCB_RESIDENT=0 the LCB as a streaming GEMM instead of with W_L resident in shared memory
  WK_GEMM_STREAM=0  the CTA-pair MLP GEMM persistent (one pair per two SMs) instead of one
                    pair per output tile
  WK_MOE_RING=0     the MoE mixture without the bulk-copy ring (runs the MoE tests)
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

VARIANTS = {
    "fused_ln": {"WK_FUSED_LN": "1"},
    "fm_mma_sync": {"WK_FM_MMA_SYNC": "1"},
    "one_cta_gemm": {"WK_PAIR_GEMM": "0"},
    "res_ln_registers": {"WK_RES_LN_RING": "0"},
    "lcb_streaming": {"WK_LCB_RESIDENT": "0"},
    "gemm_persistent": {"WK_GEMM_STREAM": "0"},
    "moe_register_combine": {"WK_MOE_RING": "0"},
}


@pytest.mark.parametrize("name", sorted(VARIANTS))
def test_variant_stack_parity(name, cuda_device):
    env = dict(os.environ, **VARIANTS[name])
    if name.startswith("moe"):
        cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_moe.py"), "-q", "-x", "-s",
               "-m", "gpu"]
    else:
        cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_stack.py"), "-q", "-x", "-s",
               "-m", "gpu", "-k", "c2_bf16 or c4_bf16 or c5_bf16 or batch_split or profiling"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    print(tail)
    assert r.returncode == 0, tail
