"""Pins on the conditioning of the workloads' recurrences (CPU, oracle only).

The TTT-MLP workload (eta_t = sigmoid(u_t)/d, LayerNorm on a 0.02-scale second
layer) is chaotic on some sequences: a 1e-7 relative change of the inputs
grows to O(1) in the outputs within the 8,192 tokens, in the exact (double)
recurrence. The same workload with a 10x smaller step stays within 1e-5, and
the linear workloads stay well conditioned. The parity tests rely on these
facts (the full-size MLP case compares each sequence up to its conditioned
horizon)."""
import numpy as np

from test_sequence_layers_layer_b200 import synth

from conditioning import conditioned_horizon, divergence

W = synth.WORKLOADS
MLP = W["mlp_ln_d64_dh256_b4h12_t8192"]
CHAOTIC_SEQ = 20  # batch 1, head 8 of the seed-0 MLP workload


def test_mlp_workload_has_a_chaotic_sequence():
    inp = synth.make_inputs(MLP)
    dev, _ = divergence(inp, seqs=[CHAOTIC_SEQ])
    assert dev[0, :1024].max() < 1e-6      # tracks at first ...
    assert dev[0].max() > 1e-2             # ... then the recurrence amplifies the change
    h, _ = conditioned_horizon(inp, seqs=[CHAOTIC_SEQ])
    assert 1024 <= h[0] < MLP.T


def test_mlp_with_smaller_step_is_well_conditioned():
    inp = synth.make_inputs(MLP.scaled(eta="sigmoid_over_d:0.1"))
    dev, _ = divergence(inp, seqs=[CHAOTIC_SEQ, 0, 42])
    assert dev.max() < 1e-5


def test_linear_long_context_is_well_conditioned():
    inp = synth.make_inputs(W["linear_ln_d64_b1h32_t32768"])
    dev, _ = divergence(inp, seqs=[0, 17])
    assert dev.max() < 1e-5
