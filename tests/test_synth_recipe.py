"""The synthetic input recipe: the generators draw what the recipe states
(shapes, distributions, outlier channels, spikes, zero blocks) and draw it
identically every time, so the oracle and the CUDA path see the same bytes."""
import numpy as np
import torch

import synth


def test_mlp_up_activations_have_one_percent_outlier_channels():
    x = synth.MLP_UP.activations()
    assert x.dtype == torch.bfloat16 and tuple(x.shape) == (4608, 3072)
    std = x.float().std(dim=0).numpy()
    outliers = np.flatnonzero(std > 5)
    assert len(outliers) == 31                       # round(1% of 3072)
    assert np.all(np.abs(std[outliers] / 20 - 1) < 0.1)
    rest = np.delete(std, outliers)
    assert np.all(np.abs(rest - 1) < 0.1)
    assert torch.equal(x, synth.MLP_UP.activations())   # same bytes on every call


def test_weights_and_bias_follow_their_normal_laws():
    wl = synth.MLP_UP
    w, b = wl.weight(), wl.bias_vec()
    assert tuple(w.shape) == (wl.n, wl.k) and tuple(b.shape) == (wl.n,)
    assert abs(float(w.float().std()) / 0.02 - 1) < 0.01
    assert abs(float(b.float().std()) / 0.01 - 1) < 0.05
    assert abs(float(w.float().mean())) < 1e-4
    assert synth.TINY.bias_vec() is None


def test_laplace_workload_has_spikes_and_zero_blocks():
    x = synth.quantize_input().float()
    assert tuple(x.shape) == (synth.QUANT_M, synth.QUANT_K)
    runs = x.view(synth.QUANT_M, -1, 16)
    zero_runs = float((runs.abs().amax(dim=2) == 0).float().mean())
    assert 0.009 < zero_runs < 0.0101                 # 1% of the runs (a few drawn twice)
    live = x[x != 0]
    assert abs(float(live.abs().median()) / np.log(2) - 1) < 0.01   # Laplace(0,1): median |x| = ln 2
    spikes = float((x.abs() > 30).float().mean())
    assert 0.0004 < spikes < 0.001                    # 0.1% spiked x50, those that land above 30


def test_sweep_and_single_stream_shapes():
    assert [w.m for w in synth.SWEEP] == [512, 1024, 4608, 9216, 16896]
    assert all((w.k, w.n) == (3072, 3072) for w in synth.SWEEP)
    assert (synth.SINGLE_IN.m, synth.SINGLE_IN.k, synth.SINGLE_IN.n) == (4608, 3072, 21504)
    assert synth.SINGLE_Q[1] == synth.SINGLE_KV[0] and synth.SINGLE_KV[1] == synth.SINGLE_MLP[0]
    assert synth.SINGLE_MLP[1] == synth.SINGLE_IN.n
    # the output projection reads [Q | GELU(MLP)]
    q = synth.SINGLE_Q[1] - synth.SINGLE_Q[0]
    mlp = synth.SINGLE_MLP[1] - synth.SINGLE_MLP[0]
    assert synth.SINGLE_OUT.k == q + mlp
