"""The whole AWQ pass over the 7B-shaped decoder layer, GPU against the oracle at every step.

The layer (seed 4: q/k/v/o [4096, 4096], gate/up [11008, 4096], down [4096, 11008]) is
calibrated on the first 1024 tokens of each of its three 65536-token calibration inputs (the
hidden state for q/k/v and gate/up, X_o for o_proj, X_d for down_proj), small enough for
the oracle to evaluate every row:

    act_stats (3 inputs) -> 4 searches over the 20-point grid (q/k/v jointly, N = 12288;
    gate/up jointly, N = 22016; o_proj; down_proj, K = 11008) -> 7 packs with the chosen
    scales -> 7 W4A16 GEMMs over the calibration tokens with inv_s = 1 / best_s.

Bars: s_x bit-exact; every loss within the search tolerance of tests/test_gpu_parity.py and
each chosen grid point equal to the oracle's unless the oracle rates the two as a near tie;
the chosen scale row equal to the oracle's power of s_x; 1 / best_s, codes, fp16 scales and
zero points bit-exact; GEMMs within 2e-3 relative Frobenius error.

robotsatlas "AWQ", "How it works" (calibration pass, per-channel scales found by a grid search
on the layer's output error, group-wise 4-bit quantization) and "Components".
"""
import multiprocessing as mp
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import pytest
import torch

import oracle as O
import synth
from test_gpu_parity import GEMM_RTOL, NEAR_TIE, assert_losses_match, cu, host_u32, rel_fro

pytestmark = pytest.mark.gpu

TOKENS = 1024
JOBS = [("hidden", ("q_proj", "k_proj", "v_proj")), ("hidden", ("gate_proj", "up_proj")),
        ("o_in", ("o_proj",)), ("down_in", ("down_proj",))]


@pytest.fixture(scope="module")
def awq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_int4_stats_b200 import build
    build.build()
    import weight_only_int4_stats_b200 as m
    return m


def test_decoder_layer_pipeline_against_oracle(awq):
    acts = synth.decoder_layer_activations(rows=TOKENS)
    Ws = synth.decoder_layer_weights()
    a = O.alpha_grid(20)
    stacked = [np.concatenate([Ws[n] for n in names]) for _, names in JOBS]

    # the oracle's four searches run in parallel processes (spawned: no CUDA state is forked)
    o_sx = {name: O.act_stats(X) for name, X in acts.items()}
    with ProcessPoolExecutor(max_workers=4, mp_context=mp.get_context("spawn")) as pool:
        futs = [pool.submit(O.search_scale, W, acts[x], o_sx[x], a, 4, 128)
                for (x, _), W in zip(JOBS, stacked)]
        ora = [f.result() for f in futs]

    # GPU: statistics -> searches -> packs -> GEMMs, all on the device
    Xd = {name: cu(X) for name, X in acts.items()}
    sx = {name: awq.awq_act_stats(X) for name, X in Xd.items()}
    for name in acts:
        np.testing.assert_array_equal(sx[name].cpu().numpy(), o_sx[name], err_msg=name)
    alphas = cu(a)
    chosen = {}
    for (x, names), W, (ol, ob, obs) in zip(JOBS, stacked, ora):
        losses, best, best_s, _, best_inv = awq.awq_search_scale(cu(W), Xd[x], sx[x], alphas, 4,
                                                                 inv=True)
        gl = losses.cpu().numpy()
        assert_losses_match(gl, ol, acts[x].shape[1], names, M=acts[x].shape[0])
        b = int(best.item())
        if b != ob:   # near tie: the oracle rates the GPU's choice within NEAR_TIE of its own
            assert ol[b] <= (1 + NEAR_TIE) * ol[ob], (names, b, ob)
        gs = best_s.cpu().numpy()
        want_s = O.scale_candidates(o_sx[x], a)[b]
        np.testing.assert_allclose(gs, want_s, rtol=2 ** -23, atol=0, err_msg=str(names))
        np.testing.assert_array_equal(best_inv.cpu().numpy(), np.float32(1.0) / gs)
        for n in names:
            chosen[n] = (x, best_s, best_inv, gs)

    for n, (x, best_s, best_inv, gs) in chosen.items():
        W = Ws[n]
        N, K = W.shape
        qw, sc, z = awq.awq_quantize_pack(cu(W), best_s, 4)
        oq, osc, oz = O.quantize_pack(W, gs, 4, 128)
        np.testing.assert_array_equal(host_u32(qw), oq, err_msg=n)
        np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint16), osc.view(np.uint16))
        np.testing.assert_array_equal(z.cpu().numpy(), oz, err_msg=n)
        Y = awq.awq_gemm_w4a16(Xd[x], qw, sc, z, N, K, 4, inv_s=best_inv)
        want = O.gemm_w4a16(acts[x], oq, osc, oz, N, K, 4, 128, inv_s=np.float32(1.0) / gs)
        err = rel_fro(Y.float().cpu().numpy(), want)
        assert err <= GEMM_RTOL, (n, err)
    torch.cuda.empty_cache()


def test_down_proj_calibrated_on_gated_mlp_output(awq):
    # down_proj's calibration input computed as a gated MLP would produce it: the GPU's
    # H = silu(X W_gate^T) * (X W_up^T) from the hidden state's first 1024 tokens and the
    # layer's fp16 gate_proj / up_proj against the oracle's; then down_proj's search on the
    # oracle's H (fp16), GPU against oracle: s_x bit-exact, losses within the search
    # tolerance, the same grid point (near ties aside), and the pack bit-exact.
    X = synth.decoder_layer_activations(names=("hidden",), rows=TOKENS)["hidden"]
    Ws = synth.decoder_layer_weights()
    Wg, Wu, Wd = Ws["gate_proj"], Ws["up_proj"], Ws["down_proj"]
    H = awq.awq_silu_mul_gemm(cu(X), cu(Wg), cu(Wu))
    want = O.silu_mul(X, Wg, Wu)
    assert rel_fro(H.float().cpu().numpy(), want) <= GEMM_RTOL
    Hh = want.astype(np.float16)                  # the oracle's H feeds both searches
    a = O.alpha_grid(20)
    o_sx = O.act_stats(Hh)
    ol, ob, obs = O.search_scale(Wd, Hh, o_sx, a, 4, 128)
    Hd = cu(Hh)
    sx = awq.awq_act_stats(Hd)
    np.testing.assert_array_equal(sx.cpu().numpy(), o_sx)
    losses, best, best_s, _ = awq.awq_search_scale(cu(Wd), Hd, sx, cu(a), 4)
    assert_losses_match(losses.cpu().numpy(), ol, Hh.shape[1], M=Hh.shape[0])
    b = int(best.item())
    if b != ob:
        assert ol[b] <= (1 + NEAR_TIE) * ol[ob], (b, ob)
    gs = best_s.cpu().numpy()
    qw, sc, z = awq.awq_quantize_pack(cu(Wd), best_s, 4)
    oq, osc, oz = O.quantize_pack(Wd, gs, 4, 128)
    np.testing.assert_array_equal(host_u32(qw), oq)
    np.testing.assert_array_equal(z.cpu().numpy(), oz)
    torch.cuda.empty_cache()
