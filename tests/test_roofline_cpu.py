"""CPU checks of the algorithmic byte and flop counts the benchmark divides by,
against the figures derived by hand from the layouts (every input read once,
every output and boundary state written once)."""
from bidirectional_mamba_state_b200 import roofline as RL
from bidirectional_mamba_state_b200 import workload as W


def test_allblock_87m_bytes():
    s = W.WORKLOADS["87m_allblock"]
    B, L, H, P, N, G, K = 16, 1024, 24, 64, 128, 1, 32
    direction = 2 * B * L * (H * P + H + 2 * G * N) + 8 * H     # bf16 x, dt, B, C; fp32 A, D
    y = 4 * B * L * H * P                                        # fp32
    states = K * 4 * B * H * P * N                               # fp32, one per block
    assert RL.allblock_bytes(s) == 4 * direction + 2 * y + states == 842_007_296


def test_block_step_and_prefill_bytes():
    st = W.WORKLOADS["700m_step"]                 # batch 1, 32 tokens, 48 heads
    state = 4 * 1 * 48 * 64 * 128
    direction = 2 * 1 * 32 * (48 * 64 + 48 + 2 * 128) + 8 * 48
    assert RL.block_step_bytes(st) == 2 * direction + 4 * 32 * 48 * 64 + state
    assert RL.block_step_bytes(st, commit=True) == RL.block_step_bytes(st) + state
    pf = W.WORKLOADS["700m_prefill_8k"]
    assert RL.prefix_bytes(pf, block_states=False) == 2 * RL.dir_bytes(pf) + RL.y_bytes(pf) + RL.state_bytes(pf)


def test_conv_and_norm_bytes():
    s = W.WORKLOADS["87m_allblock"]
    cx = 24 * 64 + 2 * 128
    per_dir = 2 * 2 * 16 * 1024 * cx + 4 * cx * (4 + 1)         # rows in and out (bf16), taps + bias
    assert RL.conv_bytes(s, 4, 4) == 4 * per_dir == 469_905_408
    st = W.WORKLOADS["700m_step"]
    assert RL.conv_bytes(st, 4, 2, state_in=True) == 2 * RL.conv_dir_bytes(st, 4) + 2 * 3 * (48 * 64 + 256)
    n = 16 * 1024 * 24 * 64
    assert RL.norm_bytes(s, gated=True) == n * (4 + 2 + 2) + 4 * 24 * 64 == 201_332_736
    assert RL.norm_bytes(s, gated=False) == n * (4 + 2) + 4 * 24 * 64


def test_allblock_flops_chunked_form():
    s = W.WORKLOADS["87m_allblock"]
    B, H, P, N, G, T, K = 16, 24, 64, 128, 1, 32, 32
    per_bhk = 2 * T * P * N + 2 * (2 * T * N * P) + 4 * (2 * T * T * P)   # S, Y_off of 2 streams, Y_diag of 4 dirs
    per_bgk = 4 * (2 * T * T * N)                                          # C B^T of 4 dirs
    assert RL.allblock_flops(s) == B * K * (H * per_bhk + G * per_bgk)
