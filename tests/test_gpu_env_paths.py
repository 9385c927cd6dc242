"""The alternative launch paths that an environment variable selects, each run
through a slice of the parity suite in a fresh process (the library reads
these variables once per process):

  MOE_PDL=0                  kernels launched without programmatic dependent
                             launch (plain stream order);
  MOE_ROUTER_TOPK=separate   tensor-core router writes logits, then the
                             standalone top-K kernel selects;
  MOE_GEMM_PATH=pair         CTA-pair (cta_group::2) expert GEMMs (bf16 and E4M3);
  MOE_GRID_BALANCE=0         persistent GEMM tiles strided over the whole grid;
  MOE_GATHER=separate/fused  the x rows gathered into Xp by their own kernel
                             before GEMM1, or by GEMM1 itself (default: by
                             GEMM1 when the experts average <= 256 rows);
  MOE_GEMM1_BAND_KB=0 / 64, MOE_GEMM2_BAND_KB=0 / 64
                             the expert GEMMs' tile order without bands, and
                             with bands of a row block or two;
  MOE_GEMM2_TILE=dual        GEMM2 on two row blocks per tile for every batch
                             (default: only when the experts average more than
                             256 rows and ffn >= 4,096);
  MOE_GEMM_PATH=dual         both GEMMs on two row blocks per tile (E4M3 here;
                             bf16 in the unit tests).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SLICE = "small and (bf16_ragged or bf16_k3_n16 or router_split2 or router_split4 or router_K10 or f32_tiny)"


@pytest.mark.parametrize("env", [{"MOE_PDL": "0"}, {"MOE_ROUTER_TOPK": "separate"}, {"MOE_GEMM_PATH": "pair"},
                                 {"MOE_GRID_BALANCE": "0"}, {"MOE_GATHER": "separate"}, {"MOE_GATHER": "fused"},
                                 {"MOE_GEMM1_BAND_KB": "0", "MOE_GEMM2_BAND_KB": "0"},
                                 {"MOE_GEMM1_BAND_KB": "64", "MOE_GEMM2_BAND_KB": "64"},
                                 {"MOE_GEMM2_TILE": "dual"}],
                         ids=lambda e: ",".join("%s=%s" % kv for kv in e.items()))
def test_parity_slice_under_env(env):
    full_env = dict(os.environ)
    full_env.update(env)
    cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"), "-m", "gpu", "-q",
           "-x", "-p", "no:cacheprovider", "-k", SLICE]
    r = subprocess.run(cmd, cwd=ROOT, env=full_env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).strip().splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "6 passed" in r.stdout, tail


@pytest.mark.parametrize("test_file,selection,count", [
    ("test_gpu_e4m3.py", "e4m3_ragged or e4m3_tails", 2),
    ("test_gpu_fp4.py", "fp4_ragged or fp4_tails", 2),
    ("test_gpu_w4a4.py", "w4a4_small or w4a4_tails", 8),    # four tile shapes
], ids=["e4m3", "fp4", "w4a4"])
def test_low_precision_paths_without_pdl(test_file, selection, count):
    """The E4M3, 4-bit and 4-bit weight-and-activation layers with plain
    stream-ordered launches (MOE_PDL=0)."""
    full_env = dict(os.environ)
    full_env["MOE_PDL"] = "0"
    cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", test_file), "-m", "gpu", "-q", "-x",
           "-p", "no:cacheprovider", "-k", selection]
    r = subprocess.run(cmd, cwd=ROOT, env=full_env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).strip().splitlines()[-15:])
    assert r.returncode == 0, tail
    assert "%d passed" % count in r.stdout, tail


@pytest.mark.parametrize("path", ["pair", "dual"])
def test_e4m3_layer_on_other_tiles(path):
    """The E4M3 layer with the CTA-pair (cta_group::2, kind::f8f6f4) GEMMs, and
    with the GEMMs on two row blocks per tile: every layer case, the capacity
    case, the 20,000-token sampled case and the full-size decode, prefill and
    skewed-prefill workloads."""
    full_env = dict(os.environ)
    full_env["MOE_GEMM_PATH"] = path
    cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_e4m3.py"), "-m", "gpu", "-q", "-x",
           "-p", "no:cacheprovider", "-k", "layer_matches_oracle or capacity or many_rows or full_size"]
    r = subprocess.run(cmd, cwd=ROOT, env=full_env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).strip().splitlines()[-15:])
    assert r.returncode == 0, tail
    assert "11 passed" in r.stdout, tail   # 6 layer cases, capacity, many rows, 3 full-size workloads
