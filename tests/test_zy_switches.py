"""The library's launch switches, read once per process from the environment:
TPB_GEMM_PAIRS=0 runs every GEMM on the one-CTA kernel (128x256 tiles) instead of CTA
pairs, TPB_PDL=0 launches without programmatic dependent launch, TPB_REDUCE_IN_GEMM=1
sums the partials inside the row GEMM instead of in a separate kernel after it,
TPB_ATTN_ONE_TILE=1 runs attention with one 128-query tile per CTA (64-key blocks, two
CTAs per SM) instead of two tiles per CTA, TPB_GEMM_WIDE=0 keeps the row layers whose
256 x 512 tiles fit one round on 256 x 256 tiles.  Each is exercised by
re-running small parity tests against the oracle in a child process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# small, every-element parity cases of the FFN (both reduce modes, fp16 W2, ragged M),
# the linears, attention (causal and not) and the layer
CASES = [
    "tests/test_gpu_ffn.py::test_bf16_small_full",
    "tests/test_gpu_ffn.py::test_bf16_sharding_invariance_bitwise_and_determinism",
    "tests/test_gpu_ffn.py::test_column_linear",
    "tests/test_gpu_ffn.py::test_row_linear",
    "tests/test_gpu_ffn.py::test_row_linear_wide_full",
    "tests/test_gpu_ffn.py::test_bf16_wide_hidden_full",
    "tests/test_gpu_ffn.py::test_row_linear_wide_two_rounds_sampled",
    "tests/test_gpu_attention_layer.py::test_attention_small_full",
    "tests/test_gpu_attention_layer.py::test_layer_small_full",
    "tests/test_gpu_backward.py::test_backward_small_full",
    "tests/test_gpu_blocks.py::test_launch_trace_names_kernels",
]


@pytest.mark.parametrize("env", [{"TPB_GEMM_PAIRS": "0"}, {"TPB_PDL": "0"}, {"TPB_REDUCE_IN_GEMM": "1"},
                                 {"TPB_ATTN_ONE_TILE": "1"}, {"TPB_GEMM_WIDE": "0"}],
                         ids=["one_cta_gemm", "no_pdl", "reduce_in_gemm", "attn_one_tile", "no_wide_tiles"])
def test_parity_under_switch(env):
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *CASES],
                       cwd=ROOT, env=dict(os.environ, **env), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
