"""Stage-isolating parity cases for the tensor-core path (bf16, d = 112, chunk 64).

Each case switches parts of the method off through its inputs, so that a
failure points at one product of the kernel:
  read_only   beta = 0, a = 1: O = S0^T q/|q|, state unchanged  (TMA q, MMA1 Q half, state copy)
  write_only  S0 = 0, a = 1: O = P E, E = T V                   (Gram, solve, U, P E)
  one_chunk   everything on, one chunk                           (W S, E, state update)
  two_chunks  state carried across a chunk boundary
  ragged      T = 200 (last chunk 8 tokens), frames of 50 tokens
"""

import numpy as np
import pytest

import hybrid_linear_attention_frame_b200 as G
from oracle import gdn_reference as R
from workloads import draw

from gpu_util import assert_bf16_parity, run_library

pytestmark = pytest.mark.gpu
BIG = 1.0e4


def make(T, seed, frame_len=64, beta_off=False, gate_one=False, zero_state=False, H=2):
    rng = np.random.Generator(np.random.PCG64(seed))
    inp = draw(rng, 1, H, T, 112, 112, frame_len, "bf16", gate_mean=0.0, gate_std=1.0,
               state_std=None if zero_state else 0.5)
    if beta_off:
        inp.beta[:] = -BIG
    if gate_one:
        inp.gate[:] = -BIG
    return inp


CASES = {
    "read_only": dict(T=64, seed=1, beta_off=True, gate_one=True),
    "write_only": dict(T=64, seed=2, gate_one=True, zero_state=True),
    "one_chunk": dict(T=64, seed=3),
    "two_chunks": dict(T=128, seed=4),
    "ragged": dict(T=200, seed=5, frame_len=50),
}


def test_tensor_core_path_selected():
    assert G.gdn_bf16_path(112, 112, 64) == 2      # the sequence-parallel kernel
    assert G.gdn_bf16_path(128, 128, 64) == 1      # d = 128: the fused kernel


@pytest.mark.parametrize("name", list(CASES))
def test_stage(cuda, name):
    inp = make(**CASES[name])
    o, s = run_library(inp, cuda, state_in=inp.state)
    ro, rs = R.token_recurrence(inp, inp.state)
    assert_bf16_parity(o, ro, name + " out")
    assert_bf16_parity(s, rs, name + " state")
