"""GPU parity of the FFN block and the parallel linears against the fp64 oracle.

Small cases compare every element; full-size workloads compare a seeded sample
of 64 token rows.  All calls go through the C-ABI (ctypes binding)."""
import os

import numpy as np
import pytest
import torch

import oracle
from megatron_tensor_transformer_bias_b200 import configs, inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import assert_bf16_close, assert_fp32_close, ffn_oracle_rows, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_ffn(inp, t, mode="fused", act="gelu", with_b1=True, with_b2=True, with_res=True, w2_fp16=False):
    X = inp["X"]
    W1s = tb.shard_columns(inp["W1"], t)
    W2s = tb.shard_rows(inputs.as_fp16(inp["W2"]) if w2_fp16 else inp["W2"], t)
    b1s = tb.shard_vector(inp["b1"], t) if with_b1 else None
    out = torch.empty_like(X)
    tb.tp_ffn_forward(X, W1s, b1s, W2s, inp["b2"] if with_b2 else None, X if with_res else None, out,
                      mode=mode, act=act)
    assert tb.tp_get_device_status() == tb.TP_OK
    return out


def _oracle_full(inp, act="gelu", with_b1=True, with_b2=True, with_res=True):
    X = to64(inp["X"])
    return oracle.ffn_forward(X, to64(inp["W1"]), to64(inp["b1"]) if with_b1 else None, to64(inp["W2"]),
                              to64(inp["b2"]) if with_b2 else None, X if with_res else None, act=act)


# ---------------------------------------------------------------- tiny fp32 workload
def test_fp32_tiny_workload_full():
    w = configs.TINY_FP32_FFN
    inp = inputs.ffn_inputs(w.M, w.h, w.f, "fp32", seed=0, device=DEV)
    out = _run_ffn(inp, w.t)
    assert out.dtype == torch.float32
    assert_fp32_close(out, _oracle_full(inp), "fp32 M8 h64 f256 t2")


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_fp32_sharding_invariance(t):
    inp = inputs.ffn_inputs(8, 64, 256, "fp32", seed=0, device=DEV)
    assert_fp32_close(_run_ffn(inp, t), _oracle_full(inp), f"fp32 t={t}")


# ---------------------------------------------------------------- small bf16 cases (every element)
SMALL = [(300, 256, 1024), (128, 128, 512), (1, 64, 256), (513, 512, 2048)]


@pytest.mark.parametrize("M,h,f", SMALL)
@pytest.mark.parametrize("t", [1, 2, 4])
@pytest.mark.parametrize("mode", ["fused", "partials"])
@pytest.mark.parametrize("w2_fp16", [False, True])
def test_bf16_small_full(M, h, f, t, mode, w2_fp16):
    inp = inputs.ffn_inputs(M, h, f, "bf16", seed=1, device=DEV)
    out = _run_ffn(inp, t, mode=mode, w2_fp16=w2_fp16)
    assert_bf16_close(out, _oracle_full(inp), f"M{M} h{h} f{f} t{t} {mode} w2_fp16={w2_fp16}")


@pytest.mark.parametrize("t", [1, 2])
def test_bf16_wide_hidden_full(t):
    """h = 10176 with M = 300: the row layer's 256 x 256 tiles (80) outnumber the CTA pairs and
    its 256 x 512 tiles (40, the last one 448 columns wide) do not, so it runs on the wide
    tiles; every element against the oracle."""
    inp = inputs.ffn_inputs(300, 10176, 256, "bf16", seed=4, device=DEV)
    out = _run_ffn(inp, t)
    assert_bf16_close(out, _oracle_full(inp), f"M300 h10176 f256 t{t}")


def test_bf16_relu_and_no_bias():
    inp = inputs.ffn_inputs(200, 256, 1024, "bf16", seed=2, device=DEV)
    out = _run_ffn(inp, 2, act="relu")
    assert_bf16_close(out, _oracle_full(inp, act="relu"), "relu")
    out = _run_ffn(inp, 4, with_b1=False, with_b2=False, with_res=False)
    assert_bf16_close(out, _oracle_full(inp, with_b1=False, with_b2=False, with_res=False), "no bias/residual")


def test_bf16_sharding_invariance_bitwise_and_determinism():
    """Fused mode sums the shards' K-slices in one accumulator in the same order
    for every t, so the output is the same bits for every t dividing f/64."""
    inp = inputs.ffn_inputs(384, 256, 2048, "bf16", seed=3, device=DEV)
    ref = _run_ffn(inp, 1)
    for t in (2, 4, 8):
        assert torch.equal(_run_ffn(inp, t), ref), f"t={t} differs from t=1"
    for mode in ("fused", "partials"):
        a = _run_ffn(inp, 4, mode=mode)
        b = _run_ffn(inp, 4, mode=mode)
        assert torch.equal(a, b), f"{mode} not deterministic"


def test_bf16_special_cases():
    inp = inputs.ffn_inputs(130, 128, 512, "bf16", seed=4, device=DEV)
    # W2 = 0: out = b2 + residual
    z = dict(inp)
    z["W2"] = torch.zeros_like(inp["W2"])
    out = _run_ffn(z, 2)
    want = (inp["X"].float() + inp["b2"].float()).to(torch.bfloat16)
    assert torch.equal(out, want)
    # X = 0 (no residual): out = GeLU(b1) W2 + b2
    z = dict(inp)
    z["X"] = torch.zeros_like(inp["X"])
    out = _run_ffn(z, 4, with_res=False)
    assert_bf16_close(out, _oracle_full(z, with_res=False), "X=0")


def test_shards_in_separate_buffers():
    """Shards need not be views of one matrix: copy each into its own buffer."""
    inp = inputs.ffn_inputs(256, 256, 1024, "bf16", seed=5, device=DEV)
    t = 4
    W1s = [w.contiguous() for w in tb.shard_columns(inp["W1"], t)]
    W2s = [w.clone() for w in tb.shard_rows(inp["W2"], t)]
    b1s = [b.clone() for b in tb.shard_vector(inp["b1"], t)]
    out = torch.empty_like(inp["X"])
    tb.tp_ffn_forward(inp["X"], W1s, b1s, W2s, inp["b2"], inp["X"], out)
    assert_bf16_close(out, _oracle_full(inp), "separate shard buffers")


# ---------------------------------------------------------------- parallel linears alone
@pytest.mark.parametrize("act", [None, "gelu", "relu"])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_column_linear(act, dt):
    M, k, n, t = 200, 256, 1024, 4
    inp = inputs.ffn_inputs(M, k, n, "bf16", seed=6, device=DEV)
    out = torch.empty(M, n, dtype=dt, device=DEV)
    tb.tp_column_linear_forward(inp["X"].to(dt), tb.shard_columns(inp["W1"].to(dt), t),
                                tb.shard_vector(inp["b1"], t), out, act=act)
    Z = to64(inp["X"]) @ to64(inp["W1"]) + to64(inp["b1"])
    ref = {None: Z, "gelu": oracle.gelu(Z) if act == "gelu" else None, "relu": oracle.relu(Z)}[act]
    assert_bf16_close(out, ref, f"column linear {act}")


@pytest.mark.parametrize("mode", ["fused", "partials"])
def test_row_linear(mode):
    M, k, n, t = 300, 1024, 256, 4
    g = torch.Generator(device=DEV).manual_seed(7)
    A = torch.randn(M, k, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(k, n, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    bias = (torch.randn(n, generator=g, device=DEV) * 0.01).to(torch.bfloat16)
    R = torch.randn(M, n, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.empty(M, n, dtype=torch.bfloat16, device=DEV)
    tb.tp_row_linear_forward(A, tb.shard_rows(W, t), bias, R, out, mode=mode)
    ref = oracle.reduce_partials([to64(A[:, i * k // t:(i + 1) * k // t]) @ to64(W[i * k // t:(i + 1) * k // t])
                                  for i in range(t)], to64(bias), to64(R))
    assert_bf16_close(out, ref, f"row linear {mode}")


# Wide fused row layers, every element checked.  Two blocks of 256 rows x 40 column tiles
# of 256 are more tiles than CTA pairs, so these run on 256 x 512 tiles in one round (with
# TPB_GEMM_WIDE=0: 256 x 256 tiles in two rounds); four blocks of rows (1024) are more
# 256 x 512 tiles than pairs too and run on 256 x 256 tiles in three rounds.  Ragged M,
# and N = 10176, which is a multiple of neither tile width.
ROW_WIDE_CASES = [(512, 256, 10240, 2), (300, 128, 10176, 1), (400, 512, 10240, 4), (1024, 128, 10176, 2)]


@pytest.mark.parametrize("M,k,n,t", ROW_WIDE_CASES)
def test_row_linear_wide_full(M, k, n, t):
    g = torch.Generator(device=DEV).manual_seed(M + n)
    A = torch.randn(M, k, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(k, n, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    bias = (torch.randn(n, generator=g, device=DEV) * 0.01).to(torch.bfloat16)
    R = torch.randn(M, n, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.full((M, n), float("nan"), dtype=torch.bfloat16, device=DEV)
    tb.tp_row_linear_forward(A, tb.shard_rows(W, t), bias, R, out, mode="fused")
    assert tb.tp_get_device_status() == tb.TP_OK
    assert torch.isfinite(out.float()).all(), "an output element was not written"
    ref = oracle.reduce_partials([to64(A[:, i * k // t:(i + 1) * k // t]) @ to64(W[i * k // t:(i + 1) * k // t])
                                  for i in range(t)], to64(bias), to64(R))
    assert_bf16_close(out, ref, f"row linear {M}x{k}x{n} t={t}")


def test_row_linear_wide_two_rounds_sampled():
    """M = 3684 (15 blocks of 256 rows, the last ragged), N = 4096, K = 8192 over t = 2: 120
    tiles of 256 x 512 take two rounds of the CTA pairs (240 tiles of 256 x 256 would take
    four), with 128 K steps per tile, so the row layer runs on wide tiles with an exposed
    epilogue between rounds.  Eight rows of every block of rows, every column, against the
    oracle; every element finite."""
    M, k, n, t = 3684, 8192, 4096, 2
    g = torch.Generator(device=DEV).manual_seed(17)
    A = torch.randn(M, k, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(k, n, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    bias = (torch.randn(n, generator=g, device=DEV) * 0.01).to(torch.bfloat16)
    R = torch.randn(M, n, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.full((M, n), float("nan"), dtype=torch.bfloat16, device=DEV)
    tb.tp_row_linear_forward(A, tb.shard_rows(W, t), bias, R, out, mode="fused")
    assert tb.tp_get_device_status() == tb.TP_OK
    assert torch.isfinite(out.float()).all(), "an output element was not written"
    rng = np.random.default_rng(17)
    rows = np.concatenate([b + rng.choice(min(256, M - b), 8, replace=False) for b in range(0, M, 256)])
    rows_t = torch.as_tensor(rows, device=DEV)
    A_s, R_s = A[rows_t], R[rows_t]
    ref = oracle.reduce_partials([to64(A_s[:, i * k // t:(i + 1) * k // t]) @ to64(W[i * k // t:(i + 1) * k // t])
                                  for i in range(t)], to64(bias), to64(R_s))
    assert_bf16_close(out[rows_t], ref, f"row linear {M}x{k}x{n} t={t}, {len(rows)} sampled rows")


ROW_PARTIAL_CASES =[(300, 384, 4), (1, 320, 2), (129, 256, 1), (513, 1024, 8), (2048, 4096, 4)]


def _row_partials_case(M, n, t):
    k = 256 * t
    g = torch.Generator(device=DEV).manual_seed(M + n + t)
    A = torch.randn(M, k, generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn(k, n, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    bias = (torch.randn(n, generator=g, device=DEV) * 0.01).to(torch.bfloat16)
    R = torch.randn(M, n, generator=g, device=DEV).to(torch.bfloat16)
    ws = tb.workspace(tb.lib().tp_row_linear_workspace_bytes(M, n, t, tb.TP_REDUCE_PARTIALS), DEV)
    out = torch.empty(M, n, dtype=torch.bfloat16, device=DEV)
    runs = []
    for _ in range(2):
        out.fill_(float("nan"))
        tb.tp_row_linear_forward(A, tb.shard_rows(W, t), bias, R, out, mode="partials", ws=ws)
        assert tb.tp_get_device_status() == tb.TP_OK
        runs.append(out.clone())
    P = ws[: t * M * n * 4].view(torch.float32).view(t, M, n)[: t - 1].clone()
    return runs, P


def test_row_partials_reduce_matches_separate_pass(tmp_path):
    """Partials mode sums the stored partials in a separate fixed-order pass; with
    TPB_REDUCE_IN_GEMM=1 (run here in a child process on the same inputs) the last shard's
    tiles add the stored partials 0..t-2 and their own inside the row GEMM, in the order
    0..t-1.  Both outputs must be the same bits, the partials 0..t-2 left in the workspace
    too, and two calls in a row must agree (the arrival counters start from zero every
    call)."""
    import subprocess
    import sys
    here = {}
    for case in ROW_PARTIAL_CASES:
        runs, P = _row_partials_case(*case)
        assert torch.equal(runs[0], runs[1]), case
        here[case] = (runs[0].cpu(), P.cpu())
    dump = tmp_path / "separate.pt"
    code = ("import sys, torch; sys.path.insert(0, %r); from tests import test_gpu_ffn as T; "
            "torch.save({c: tuple(x.cpu() for x in (T._row_partials_case(*c)[0][0], T._row_partials_case(*c)[1])) "
            "for c in T.ROW_PARTIAL_CASES}, %r)" % (ROOT, str(dump)))
    r = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, TPB_REDUCE_IN_GEMM="1"),
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    there = torch.load(dump)
    for case in ROW_PARTIAL_CASES:
        assert torch.equal(here[case][0], there[case][0]), f"output {case}"
        assert torch.equal(here[case][1], there[case][1]), f"partials {case}"


# ---------------------------------------------------------------- full-size workloads (sampled rows)
@pytest.fixture(scope="module")
def ffn_2048():
    w = configs.ffn_2048x4096x16384(4)
    inp = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=DEV)
    rows = inputs.sample_rows(w.M, configs.SAMPLED_ROWS, seq=w.seq)
    ref = ffn_oracle_rows(inp, rows)
    yield inp, rows, ref
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("t", configs.FFN_SHARD_COUNTS)
@pytest.mark.parametrize("mode", ["fused", "partials"])
@pytest.mark.parametrize("w2_fp16", [False, True])
def test_ffn_2048x4096x16384_sampled(ffn_2048, t, mode, w2_fp16):
    inp, rows, ref = ffn_2048
    out = _run_ffn(inp, t, mode=mode, w2_fp16=w2_fp16)
    assert_bf16_close(out[rows], ref, f"M2048 h4096 f16384 t{t} {mode} w2_fp16={w2_fp16}")
    # properties that hold at every row: finite, and fused output bit-identical across t
    assert torch.isfinite(out.float()).all()


def test_ffn_2048_bitwise_across_t(ffn_2048):
    inp, _, _ = ffn_2048
    ref = _run_ffn(inp, 1)
    for t in (2, 4, 8):
        assert torch.equal(_run_ffn(inp, t), ref)


@pytest.mark.parametrize("h", configs.SWEEP_HIDDEN)
def test_ffn_hidden_sweep_sampled(h):
    """The sweep runs with fp16 W2 (act(Z) stored in fp16): with bf16 act(Z) the output's
    rounding noise grows with sqrt(f) and passes the 3e-2 absolute floor of the element
    bound only up to h ~ 6144 (output std ~ 12.7 at h = 22528)."""
    M = 4096
    inp = inputs.ffn_inputs(M, h, 4 * h, "bf16", seed=0, device=DEV)
    rows = inputs.sample_rows(M, configs.SAMPLED_ROWS)
    ref = ffn_oracle_rows(inp, rows, chunks=16)
    for t in configs.SWEEP_SHARDS:
        out = _run_ffn(inp, t, w2_fp16=True)
        assert_bf16_close(out[rows], ref, f"M4096 h{h} t{t}")
    del inp, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("h", [8192, 22528])
def test_ffn_hidden_sweep_bf16_w2_error_recorded(h):
    """The same sweep points with bf16 W2 (act(Z) stored in bf16), the deviation the
    fp16 copy avoids.  Records the measured error against the oracle (printed with
    the prefix RECORD); asserts only the relative Frobenius bound, which holds, while
    the per-element bound 3e-2 + 2e-2|ref| is what bf16 act(Z) breaks at these sizes."""
    from tests.parity import errors
    M = 4096
    inp = inputs.ffn_inputs(M, h, 4 * h, "bf16", seed=0, device=DEV)
    rows = inputs.sample_rows(M, configs.SAMPLED_ROWS)
    ref = ffn_oracle_rows(inp, rows, chunks=16)
    for t in configs.SWEEP_SHARDS:
        out = _run_ffn(inp, t, w2_fp16=False)
        rel_fro, excess, maxabs = errors(out[rows], ref)
        out16 = _run_ffn(inp, t, w2_fp16=True)
        rel16, excess16, maxabs16 = errors(out16[rows], ref)
        print(f"RECORD sweep h={h} t={t}: bf16 act(Z) rel_fro={rel_fro:.3e} max|err|={maxabs:.3e} "
              f"element_excess={excess:.3e}; fp16 act(Z) rel_fro={rel16:.3e} max|err|={maxabs16:.3e} "
              f"element_excess={excess16:.3e}")
        assert rel_fro <= 5e-3
        assert excess16 <= 0
    del inp, out, out16
    torch.cuda.empty_cache()


def test_column_gelu_closed_forms_identity_weights():
    """With W1 = I and no bias the column layer's epilogue output is GeLU(X) element by
    element (fp16 operands and output): GeLU(0) = 0, table values of z * Phi(z),
    GeLU(z) - GeLU(-z) = z, GeLU(z) = z and GeLU(-z) = 0 far in the tails."""
    h, t = 256, 2
    g = torch.Generator(device=DEV).manual_seed(23)
    z = torch.randn(64, h // 2, generator=g, device=DEV) * 3
    table = torch.tensor([0.0, 1.0, 2.0, 0.5, 16.0], device=DEV)
    z[0, :5] = table
    X = torch.cat([z, -z], dim=1).to(torch.float16)       # columns j and j + h/2 hold z and -z
    W = torch.eye(h, device=DEV).to(torch.float16)
    out = torch.empty(64, h, dtype=torch.float16, device=DEV)
    tb.tp_column_linear_forward(X, tb.shard_columns(W, t), None, out, act="gelu")
    got = to64(out)
    x = to64(X)
    assert got[0, 0] == 0.0 and got[0, h // 2] == 0.0
    ulp = 2.0 ** -10
    for col, phi in [(1, 0.8413447460685429), (2, 0.9772498680518208), (3, 0.6914624612740131)]:
        want = x[0, col] * phi
        assert abs(got[0, col] - want) <= ulp * abs(want), (col, got[0, col], want)
    assert got[0, 4] == 16.0 and got[0, 4 + h // 2] == 0.0
    half = h // 2
    # odd part: GeLU(z) - GeLU(-z) = z, each side rounded once to fp16
    d = got[:, :half] - got[:, half:]
    assert np.all(np.abs(d - x[:, :half]) <= ulp * (np.abs(got[:, :half]) + np.abs(got[:, half:])) + 1e-7)
    ref = oracle.gelu(x)
    assert np.all(np.abs(got - ref) <= ulp * np.abs(ref) + 1e-7)
