"""GPU parity of the packed ragged-sequence entry points (cu_seqlens) against
the fp64 oracle, which solves every sequence on its own.

Lengths mix empty sequences, single steps, sequences shorter than a tile and
sequences that cross several 32-step tiles, so that tiles start and end in
the middle of sequences and several sequences start inside one tile.  d = 40
takes the TMA tile path, d = 33 and d = 18 the cp.async one.  Tolerances as
in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import Workload, as_f64, make_inputs

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4


def _dev(t):
    return None if t is None else t.to("cuda").contiguous()


def _case(lengths, d, d_in, dtype, forget, seed):
    """Packed inputs: x (total_T, d_in), W_x, bias, R, dH (total_T, d), s0 (n, 4, d), cu (n + 1,)."""
    total = int(sum(lengths))
    w = Workload("v", 1, total, d_in, d, dtype, forget, 0.5, seed, 1e-6, 64)
    inp = make_inputs(w, with_dH=True)
    g = torch.Generator().manual_seed(seed + 1000)
    n = len(lengths)
    s0 = torch.stack([torch.randn(n, d, generator=g), torch.rand(n, d, generator=g) + 0.5,
                      torch.randn(n, d, generator=g), torch.rand(n, d, generator=g) - 0.5], dim=1)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return {"x": inp["x"][0], "Wx": inp["Wx"], "bias": inp["bias"], "R": inp["R"], "dH": inp["dH"][0],
            "s0": s0, "cu": cu}


def _preact(c):
    P = api.preact_gemm(_dev(c["x"])[None], _dev(c["Wx"]), _dev(c["bias"]))[0].contiguous()
    Pref = oracle.preact(as_f64(c["x"])[None], as_f64(c["Wx"]), as_f64(c["bias"]))[0]
    return P, Pref


def _h_err(S_gpu, S_ref):
    h = S_ref[:, 3, :]
    return float((np.abs(S_gpu[:, 3, :] - h) / (1 + np.abs(h))).max())


LENGTHS = [[5, 0, 1, 40, 33, 64, 7, 0], [70, 3], [32, 32, 32], [1, 1, 1, 1, 1], [17]]


# carry modes: 1 = one fused launch per iteration (decoupled look-back),
# 2 = two passes with a scan of tile aggregates in between
CARRY_MODES = [1, 2]


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("d", [40, 33])
@pytest.mark.parametrize("lengths", LENGTHS)
def test_varlen_fixed_k_matches_oracle(lengths, d, forget, carry_mode, cuda_device):
    K = 3
    c = _case(lengths, d, 12, "f32", forget, 41)
    P, Pref = _preact(c)
    S, st = api.newton_forward_varlen(P, _dev(c["R"]), _dev(c["s0"]), _dev(c["cu"]), forget=forget, max_iters=K,
                                      fixed=True, tol=1e-6, carry_mode=carry_mode)
    torch.cuda.synchronize()
    got = as_f64(S.cpu())
    assert api.read_stats(st)["iters"] == K
    # The whole iterate after K iterations from the decoupled guess of every
    # sequence, against the fp64 iterate of each sequence on its own.
    ref = oracle.newton_varlen_fixed(Pref, as_f64(c["R"]), as_f64(c["s0"]), c["cu"].numpy(), forget, K,
                                     sweeps=api.DEFAULT_GUESS_SWEEPS)
    assert float((np.abs(got - ref) / (1 + np.abs(ref))).max()) <= TOL_F32
    # Newton's prefix exactness, per sequence: after K iterations the first K
    # steps of every sequence are the sequential trajectory; a carry leaking
    # across a sequence start would break it.
    seq = oracle.sequential_varlen(Pref, as_f64(c["R"]), as_f64(c["s0"]), c["cu"].numpy(), forget)
    cu = c["cu"].numpy()
    for k in range(len(lengths)):
        a = int(cu[k])
        b = min(int(cu[k + 1]), a + K)
        if b > a:
            assert _h_err(got[a:b], seq[a:b]) <= TOL_F32, (k, a, b)


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("d", [40, 33])
def test_varlen_converges_to_sequential(d, carry_mode, cuda_device):
    lengths = [12, 0, 1, 40, 33, 9]
    c = _case(lengths, d, 16, "f32", "sigmoid", 42)
    P, Pref = _preact(c)
    S, st = api.newton_forward_varlen(P, _dev(c["R"]), _dev(c["s0"]), _dev(c["cu"]), max_iters=64, tol=1e-6,
                                      carry_mode=carry_mode)
    torch.cuda.synchronize()
    s = api.read_stats(st)
    assert s["error"] == 0 and s["converged"], s
    ref = oracle.sequential_varlen(Pref, as_f64(c["R"]), as_f64(c["s0"]), c["cu"].numpy())
    assert _h_err(as_f64(S.cpu()), ref) <= TOL_F32


def test_varlen_equal_lengths_matches_batched(cuda_device):
    B, T, d = 3, 50, 40
    c = _case([T] * B, d, 16, "f32", "sigmoid", 43)
    P, _ = _preact(c)
    R, s0 = _dev(c["R"]), _dev(c["s0"])
    # converged solutions (packed and batched tiles round in different orders)
    Sv, stv = api.newton_forward_varlen(P, R, s0, _dev(c["cu"]), max_iters=64, tol=1e-6)
    Sb, stb = api.newton_forward(P.view(B, T, 4, d), R, s0, max_iters=64, tol=1e-6)
    torch.cuda.synchronize()
    assert api.read_stats(stv)["converged"] and api.read_stats(stb)["converged"]
    a, b = as_f64(Sv.cpu()).reshape(B, T, 4, d), as_f64(Sb.cpu())
    assert float((np.abs(a - b) / (1 + np.abs(b))).max()) <= TOL_F32


@pytest.mark.parametrize("bad", [[0, 5, 3, 10], [0, 4, 9], [1, 4, 10]])
def test_varlen_malformed_offsets_report_invalid_arg(bad, cuda_device):
    total, d = 10, 8
    c = _case([total], d, 8, "f32", "sigmoid", 44)
    P, _ = _preact(c)
    cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
    n = len(bad) - 1
    s0 = torch.zeros(n, 4, d, device="cuda")
    S = torch.full_like(P, float("nan"))
    S, st = api.newton_forward_varlen(P, _dev(c["R"]), s0, cu, max_iters=3, S=S)
    torch.cuda.synchronize()
    s = api.read_stats(st)
    assert s["error"] == 1 and s["iters"] == 0, s     # SLSTM_ERR_INVALID_ARG, nothing ran
    assert torch.isnan(S).all()                       # S untouched


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("d_in,d,dtype", [(12, 40, "f32"), (16, 40, "bf16"), (16, 18, "bf16")])
def test_varlen_backward_matches_oracle(d_in, d, dtype, forget, cuda_device):
    lengths = [5, 0, 1, 40, 33, 36, 7, 0]
    c = _case(lengths, d, d_in, dtype, forget, 45)
    P, Pref = _preact(c)
    cu = c["cu"].numpy()
    Sref = oracle.sequential_varlen(Pref, as_f64(c["R"]), as_f64(c["s0"]), cu, forget)
    S = torch.from_numpy(Sref).float().cuda()
    out = api.newton_backward_varlen(_dev(c["x"]), _dev(c["Wx"]), P, _dev(c["R"]), _dev(c["s0"]), _dev(c["cu"]),
                                     S, _dev(c["dH"]), forget=forget)
    torch.cuda.synchronize()
    ref = oracle.backward_varlen(as_f64(c["x"]), as_f64(c["Wx"]), Pref, as_f64(c["R"]), as_f64(c["s0"]), Sref,
                                 as_f64(c["dH"]), cu, forget)
    for k in ("dx", "dWx", "dR", "db", "ds0"):
        got = as_f64(out[k].cpu())
        err = np.abs(got - ref[k]).max() / (1 + np.abs(ref[k]).max())
        assert err <= 1e-4, (k, err)
    # empty sequences get exactly zero
    assert not out["ds0"][1].any() and not out["ds0"][7].any()


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
def test_varlen_nan_in_one_sequence_reports_divergence(carry_mode, cuda_device):
    """A non-finite value inside a short sequence does not leak into the next
    sequence (its start ignores the state before it), so the steps after it in
    the same thread are finite again; the residual maximum must still keep the
    NaN and the run must report divergence."""
    lengths = [2, 3, 40]
    c = _case(lengths, 40, 12, "f32", "sigmoid", 46)
    P, _ = _preact(c)
    P[0, 1, 5] = float("nan")    # first sequence, step 0, gate i of feature 5
    S, st = api.newton_forward_varlen(P, _dev(c["R"]), _dev(c["s0"]), _dev(c["cu"]), max_iters=2, fixed=True,
                                      tol=1e-6, carry_mode=carry_mode)
    torch.cuda.synchronize()
    s = api.read_stats(st)
    assert s["diverged"] and s["error"] == 3, s
    # the later sequences are untouched by it
    assert torch.isfinite(S[2:]).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_backward_two_pass_matches_oracle(dtype, cuda_device):
    """Few feature groups and a long packed axis: the adjoint takes the two
    passes (tile aggregates, blocked scan, then the fused pass with known
    carries) instead of the look-back."""
    lengths = [5000, 0, 3000, 7000, 1700]
    d = 40
    c = _case(lengths, d, 16, dtype, "sigmoid", 47)
    P, Pref = _preact(c)
    cu = c["cu"].numpy()
    Sref = oracle.sequential_varlen(Pref, as_f64(c["R"]), as_f64(c["s0"]), cu, "sigmoid")
    S = torch.from_numpy(Sref).float().cuda()
    out = api.newton_backward_varlen(_dev(c["x"]), _dev(c["Wx"]), P, _dev(c["R"]), _dev(c["s0"]), _dev(c["cu"]),
                                     S, _dev(c["dH"]), forget="sigmoid")
    torch.cuda.synchronize()
    ref = oracle.backward_varlen(as_f64(c["x"]), as_f64(c["Wx"]), Pref, as_f64(c["R"]), as_f64(c["s0"]), Sref,
                                 as_f64(c["dH"]), cu, "sigmoid")
    for k in ("dx", "dWx", "dR", "db", "ds0"):
        got = as_f64(out[k].cpu())
        err = np.abs(got - ref[k]).max() / (1 + np.abs(ref[k]).max())
        assert err <= 1e-4, (k, err)
    assert not out["ds0"][1].any()
