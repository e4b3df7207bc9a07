"""Seeded synthetic inputs (weights, predictors, thresholds, token vectors).

Shared by the oracle tests, the GPU parity tests and the benchmark.  It holds no
arithmetic of the sparse FFN itself; see `generate` for the readings it encodes.
"""
from .workloads import (Workload, FFN512_LIT, FFN512_CAL, LLAMA2_7B, LLAMA2_7B_ADAPTIVE, FALCON_40B,
                        LLAMA2_70B_Q4, OPT_175B, ALL, adaptive_ranks, scaled)
from .generate import (SynthLayer, make_layer, make_inputs, firing_probs,
                       powerlaw_by_rank, calibrate_c, law_constant,
                       calibration_inputs, seed_of, torch_gen)
